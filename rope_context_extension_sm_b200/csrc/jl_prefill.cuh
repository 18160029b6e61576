// jl_prefill.cuh -- bifocal prefill attention on sm_100a (tcgen05 + TMEM + TMA).
//
// Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
// RoPE", Methodology section 1 (local window w0 with classical RoPE, remote map
// f(x) = floor(x/G), G = max(1, ceil(L/w_pretrained))) and section 2 (three
// flash-style passes merged by inclusion-exclusion on their log-sum-exp
// statistics).
//
// How the three passes are realised.  Pass 1 (local window, base positions)
// touches only key tiles that hold a pair with i - j < w0.  Pass 2 (causal,
// remote positions) minus pass 3 (local window, remote positions) is, tile by
// tile, pass 2 restricted to pairs with i - j >= w0, so it is evaluated with
// that mask *before* accumulation instead of being subtracted afterwards (equal
// in exact arithmetic; no cancellation of Z2 - Z3).  Both share one online
// softmax state per row; the running (max, sum) rescale between them is the
// log-sum-exp merge, finalised in the epilogue (out = O / l, lse = m + log l).
// Tiles entirely inside the window run only pass 1, tiles entirely outside run
// only pass 2 - 3, and only the (at most two) tiles per row block that straddle
// the window edge run both.  G = 1 (L <= w_pretrained) makes remote scores equal
// base scores, so every tile runs as pass 1 without any distance mask.
//
// CTA = one 128-row query block of one sequence x NQT query heads that share a
// KV head (GQA).  Each K/V tile is loaded once by TMA and feeds all NQT heads.
//   warp 0      TMA producer (Q, K, V tiles; 128B-swizzled boxes)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-3   in-place RoPE rotation of the Q and K tiles in shared memory
//               (base rows R(x) or remote rows R(f(x)), from the fp32 tables)
//   warps 4..   one warpgroup per query head: softmax on S read from TMEM,
//               P written back to TMEM (bf16), O rescale, epilogue
// TMEM columns: S_t at 128 t, O_t at 128 NQT + D t; P_t aliases S_t.
// With NQT = 2 the MMA issue order S0(n), PV1(n-1), S1(n), PV0(n) lets one
// head's softmax overlap the other head's tensor-core work.
#pragma once

#include "jl_device.cuh"

namespace jl {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kStages = 2;

struct PrefillParams {
  const int32_t* cu_seqlens;
  const float* cos_tab;
  const float* sin_tab;
  __nv_bfloat16* out;
  float* lse;
  int64_t total_tokens;
  int64_t n_tab_rows;
  int32_t batch;
  int32_t n_qtiles;      // ceil(max_seqlen / 128)
  int32_t Hq;
  int32_t Hkv;
  int32_t group;         // Hq / Hkv
  int32_t slots;         // group / NQT
  int32_t w0;
  int32_t w_pre;
  int32_t plain;
  float scale_log2;      // softmax scale * log2(e)
};

template <int D, int NQT>
struct PrefillLayout {
  static constexpr int kTileBytes = kBM * D * 2;  // 128 rows x D bf16 (Q, K or V tile)
  static constexpr int kBoxBytes = 128 * 128;     // one 128-row x 64-col box
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + NQT * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
  static constexpr int kColsUsed = NQT * 128 + NQT * D;
  static constexpr uint32_t kTmemCols = kColsUsed <= 256 ? 256u : 512u;
  static constexpr int kThreads = 128 + NQT * 128;
};

struct PrefillBars {
  uint64_t q_full, q_ready, q_empty;
  uint64_t k_full[kStages], k_ready[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_ready[2], o_final[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

// Which key tiles a query block visits and in which order.
struct TileSchedule {
  int q_lo, q_hi;  // first / last valid query position of the block
  int n_kt;        // key tiles 0 .. n_kt-1 hold causal pairs
  int R;           // remote tiles: kt in [0, R)   (hold a pair with i - j >= w0)
  int Lo;          // local tiles:  kt in [Lo, n_kt) (hold a pair with i - j <  w0)
  int n_virt;      // R + (n_kt - Lo): remote visits first, then local visits
  int w0;          // effective window (huge when every pair is local)

  __device__ void init(int qt, int L, int w0_eff) {
    w0 = w0_eff;
    q_lo = qt * kBM;
    q_hi = min(q_lo + kBM - 1, L - 1);
    n_kt = q_hi / kBN + 1;
    R = (q_hi >= w0) ? min(n_kt, (q_hi - w0) / kBN + 1) : 0;
    if (w0 <= 0) {
      Lo = n_kt;
    } else {
      const int x = q_lo - (kBN - 1) - w0;  // local iff kt * 128 > x
      Lo = (x < 0) ? 0 : min(n_kt, x / kBN + 1);
    }
    n_virt = R + (n_kt - Lo);
  }
  __device__ bool remote(int n) const { return n < R; }
  __device__ int kt(int n) const { return n < R ? n : Lo + (n - R); }
  // Does visit n need a per-element mask (window edge or causal diagonal)?
  __device__ bool masked(int n) const {
    const int k = kt(n);
    const bool diag = k * kBN + kBN - 1 > q_lo;
    return diag || (n < R ? (k >= Lo) : (k < R));
  }
};

// Rotate one 128-byte-swizzled row of a [128 rows][D] bf16 tile in place by R(p).
// Lane l owns frequency pairs c in [l*FPL, l*FPL + FPL) with partners c + D/2.
template <int D>
__device__ __forceinline__ void rotate_row_inplace(uint8_t* tile, int r, const float* __restrict__ cos_row,
                                                   const float* __restrict__ sin_row, int lane) {
  if constexpr (D == 128) {
    // elements 2l, 2l+1 (box 0) and 64+2l, 64+2l+1 (box 1), same swizzled offset
    const int off = r * 128 + ((((lane >> 2) ^ (r & 7))) << 4) + ((lane & 3) << 2);
    __nv_bfloat162* plo = reinterpret_cast<__nv_bfloat162*>(tile + off);
    __nv_bfloat162* phi = reinterpret_cast<__nv_bfloat162*>(tile + 16384 + off);
    const float2 cs = *reinterpret_cast<const float2*>(cos_row + 2 * lane);
    const float2 sn = *reinterpret_cast<const float2*>(sin_row + 2 * lane);
    const float2 a = __bfloat1622float2(*plo);
    const float2 b = __bfloat1622float2(*phi);
    float2 ya, yb;
    ya.x = a.x * cs.x - b.x * sn.x;
    yb.x = b.x * cs.x + a.x * sn.x;
    ya.y = a.y * cs.y - b.y * sn.y;
    yb.y = b.y * cs.y + a.y * sn.y;
    *plo = __float22bfloat162_rn(ya);
    *phi = __float22bfloat162_rn(yb);
  } else {
    // D == 64: element l and l + 32 of the single box
    const int c0 = lane, c1 = lane + 32;
    const int off0 = r * 128 + ((((c0 * 2) >> 4) ^ (r & 7)) << 4) + ((c0 * 2) & 15);
    const int off1 = r * 128 + ((((c1 * 2) >> 4) ^ (r & 7)) << 4) + ((c1 * 2) & 15);
    __nv_bfloat16* pa = reinterpret_cast<__nv_bfloat16*>(tile + off0);
    __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(tile + off1);
    const float cs = cos_row[lane], sn = sin_row[lane];
    const float a = __bfloat162float(*pa), b = __bfloat162float(*pb);
    *pa = __float2bfloat16_rn(a * cs - b * sn);
    *pb = __float2bfloat16_rn(b * cs + a * sn);
  }
}

// Rotate rows r = r0, r0 + stride, ... of a tile whose row r sits at position base + r.
template <int D>
__device__ __forceinline__ void rotate_tile(uint8_t* tile, int r0, int stride, int base, bool remote, int G,
                                            const PrefillParams& p, int lane) {
  constexpr int HALF = D / 2;
  const int64_t max_row = p.n_tab_rows - 1;
#pragma unroll 4
  for (int r = r0; r < kBM; r += stride) {
    int pos = base + r;
    int64_t row = remote ? (pos / G) : pos;
    row = row > max_row ? max_row : row;  // rows past the sequence end are masked later
    rotate_row_inplace<D>(tile, r, p.cos_tab + row * HALF, p.sin_tab + row * HALF, lane);
  }
}

template <int D, int NQT>
__global__ void __launch_bounds__(PrefillLayout<D, NQT>::kThreads, 1)
    jl_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using Lay = PrefillLayout<D, NQT>;
  constexpr int NBOX = D / 64;                 // 64-column boxes per tile
  constexpr uint32_t kTileTx = kBM * D * 2;    // bytes per tile load
  constexpr int KSTEPS = D / 16;               // k-steps of S = Q K^T
  constexpr int PSTEPS = kBN / 16;             // k-steps of O += P V
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, false, true);

  // ---- work item (heaviest query blocks first) ----
  const int per = p.batch * p.Hkv * p.slots;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / per;
  const int rem = static_cast<int>(blockIdx.x) % per;
  const int b = rem / (p.Hkv * p.slots);
  const int hkv = (rem / p.slots) % p.Hkv;
  const int slot = rem % p.slots;
  const int h0 = hkv * p.group + slot * NQT;
  const int seq0 = p.cu_seqlens[b];
  const int L = p.cu_seqlens[b + 1] - seq0;
  if (qt * kBM >= L) return;  // uniform across the CTA, before any barrier exists
  if (status_failed()) return;

  int G = 1;
  if (!p.plain) G = max(1, (L + p.w_pre - 1) / p.w_pre);
  const int w0_eff = (p.plain || G == 1) ? (1 << 30) : p.w0;
  TileSchedule sc;
  sc.init(qt, L, w0_eff);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem + Lay::kQ;
  uint8_t* sK = smem + Lay::kK;
  uint8_t* sV = smem + Lay::kV;
  PrefillBars* bars = reinterpret_cast<PrefillBars*>(smem + Lay::kBar);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_ready, 2);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_ready[s], 2);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_ready[t], 128);
      mbar_init(&bars->o_final[t], 1);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued_q = 0;
      int issued[kStages] = {0};
      for (int n = 0; n < sc.n_virt && !*abort; ++n) {
        if (n == 0 || n == sc.R) {
          if (n > 0 && !mbar_wait(&bars->q_empty, 0, abort)) break;
          mbar_arrive_expect_tx(&bars->q_full, kTileTx * NQT);
          for (int t = 0; t < NQT; ++t)
            for (int bx = 0; bx < NBOX; ++bx)
              tma_load_3d(sQ + t * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_q, &bars->q_full, bx * 64, h0 + t,
                          seq0 + sc.q_lo);
          ++issued_q;
        }
        const int s = n % kStages;
        const uint32_t u = n / kStages;
        const int key0 = seq0 + sc.kt(n) * kBN;
        if (u > 0 && !mbar_wait(&bars->k_empty[s], (u - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], kTileTx);
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(sK + s * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_k, &bars->k_full[s], bx * 64, hkv, key0);
        if (u > 0 && !mbar_wait(&bars->v_empty[s], (u - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], kTileTx);
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(sV + s * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_v, &bars->v_full[s], bx * 64, hkv, key0);
        issued[s] = static_cast<int>(u) + 1;
      }
      // Drain: never leave the CTA with a bulk copy still landing in its shared memory.
      if (issued_q > 0) mbar_wait_bounded(&bars->q_full, (issued_q - 1) & 1);
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0) {
          mbar_wait_bounded(&bars->k_full[s], (issued[s] - 1) & 1);
          mbar_wait_bounded(&bars->v_full[s], (issued[s] - 1) & 1);
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      auto issue_s = [&](int t, int s) {
        const uint32_t qa = q_addr + t * Lay::kTileBytes;
        const uint32_t ka = k_addr + s * Lay::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + t * 128, sdesc_kmajor_sw128(qa + off), sdesc_kmajor_sw128(ka + off), kIdescS, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int s, bool acc) {
        const uint32_t va = v_addr + s * Lay::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < PSTEPS; ++kk)
          umma_ts(tmem + NQT * 128 + t * D, tmem + t * 128 + kk * 8, sdesc_mnmajor_sw128(va + kk * 2048, 16384),
                  kIdescO, (acc || kk > 0) ? 1u : 0u);
      };
      int n = 0;
      bool ok = true;
      for (; n < sc.n_virt && ok; ++n) {
        if (n == 0 || n == sc.R) {
          if (!(ok = mbar_wait(&bars->q_ready, n == 0 ? 0 : 1, abort))) break;
          tc_fence_after();
        }
        const int s = n % kStages;
        const uint32_t u = n / kStages;
        if (!(ok = mbar_wait(&bars->k_ready[s], u & 1, abort))) break;
        tc_fence_after();
        issue_s(0, s);
        umma_commit(&bars->s_full[0]);
        if (NQT == 2) {
          if (n > 0) {
            const int sp = (n - 1) % kStages;
            if (!(ok = mbar_wait(&bars->p_ready[1], (n - 1) & 1, abort))) break;
            tc_fence_after();
            if (!(ok = mbar_wait(&bars->v_full[sp], ((n - 1) / kStages) & 1, abort))) break;
            issue_pv(1, sp, n - 1 > 0);
            umma_commit(&bars->v_empty[sp]);
          }
          issue_s(1, s);
          umma_commit(&bars->s_full[1]);
        }
        umma_commit(&bars->k_empty[s]);
        if (n == sc.R - 1 && sc.R < sc.n_virt) umma_commit(&bars->q_empty);
        if (!(ok = mbar_wait(&bars->p_ready[0], n & 1, abort))) break;
        tc_fence_after();
        if (!(ok = mbar_wait(&bars->v_full[s], u & 1, abort))) break;
        issue_pv(0, s, n > 0);
        if (NQT == 1) umma_commit(&bars->v_empty[s]);
      }
      if (ok && NQT == 2) {
        const int nl = sc.n_virt - 1;
        const int sl = nl % kStages;
        ok = mbar_wait(&bars->p_ready[1], nl & 1, abort);
        if (ok) {
          tc_fence_after();
          ok = mbar_wait(&bars->v_full[sl], (nl / kStages) & 1, abort);
        }
        if (ok) {
          issue_pv(1, sl, nl > 0);
          umma_commit(&bars->v_empty[sl]);
        }
      }
      if (ok) {
        umma_commit(&bars->o_final[0]);
        if (NQT == 2) umma_commit(&bars->o_final[1]);
      }
      // Every issued MMA must finish before TMEM is released.
      umma_commit(&bars->teardown);
      mbar_wait_bounded(&bars->teardown, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ rotation
    const int rw = warp - 2;
    for (int n = 0; n < sc.n_virt; ++n) {
      const bool remote = sc.remote(n);
      if (n == 0 || n == sc.R) {
        if (!mbar_wait(&bars->q_full, n == 0 ? 0 : 1, abort)) break;
        for (int t = 0; t < NQT; ++t)
          rotate_tile<D>(sQ + t * Lay::kTileBytes, rw, 2, sc.q_lo, remote, G, p, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_ready);
      }
      const int s = n % kStages;
      if (!mbar_wait(&bars->k_full[s], (n / kStages) & 1, abort)) break;
      rotate_tile<D>(sK + s * Lay::kTileBytes, rw, 2, sc.kt(n) * kBN, remote, G, p, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->k_ready[s]);
    }
  } else {
    // ------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;  // query head slot
    const int wq = warp & 3;        // TMEM lane quarter
    const int row = wq * 32 + lane;
    const int i = sc.q_lo + row;    // query position
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t t_s = t_lane + t * 128;
    const uint32_t t_o = t_lane + NQT * 128 + t * D;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;  // running max of scaled scores (log2 units)
    float l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < sc.n_virt; ++n) {
      if (!(ok = mbar_wait(&bars->s_full[t], n & 1, abort))) break;
      tc_fence_after();
      // Pass A: row max over the (masked) scores, 32 columns at a time.
      const bool msk = sc.masked(n);
      const int hi = i - sc.kt(n) * kBN;  // causal: keep column c <= hi
      const int edge = hi - sc.w0;        // remote keeps c <= edge, local keeps c > edge
      const bool rem = sc.remote(n);
      const int keep_lo = msk ? (rem ? -1 : edge) : -1;     // keep c > keep_lo
      const int keep_hi = msk ? (rem ? edge : hi) : kBN;    // keep c <= keep_hi
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t sr[32];
        tmem_ld32(t_s + c * 32, sr);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = c * 32 + e;
          const float x = __uint_as_float(sr[e]);
          mx = (col > keep_lo && col <= keep_hi) ? fmaxf(mx, x) : mx;
        }
      }
      const float m_new = fmaxf(m_run, mx * sl2);
      // Lazy rescale: keep the stale max unless the new one exceeds it by > 8 (x256).
      const bool resc = (m_run != -INFINITY) && (m_new > m_run + 8.f);
      const float alpha = resc ? ex2_approx(m_run - m_new) : 1.f;
      if (resc || m_run == -INFINITY) m_run = m_new;
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // Pass B: P = 2^(s * scale_log2 - m), written back over S as bf16 pairs.
      // Chunk c reads S columns [32c, 32c+32) and writes P columns [16c, 16c+16);
      // every write lands on S columns that were already read.
      float lsum = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t sr[32];
        tmem_ld32(t_s + c * 32, sr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int col = c * 32 + 2 * e;
          float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * e]), sl2, -m_use));
          float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * e + 1]), sl2, -m_use));
          p0 = (col > keep_lo && col <= keep_hi) ? p0 : 0.f;
          p1 = (col + 1 > keep_lo && col + 1 <= keep_hi) ? p1 : 0.f;
          lsum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        // 16 packed words = keys 32c .. 32c+31 -> columns 128 t + 16 c .. + 15 (P_t aliases S_t)
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15, %16};\n" ::"r"(t_s + c * 16),
            "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]), "r"(pk[7]),
            "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]), "r"(pk[12]), "r"(pk[13]), "r"(pk[14]), "r"(pk[15])
            : "memory");
      }
      l_run = l_run * alpha + lsum;
      // O_t *= alpha for the rows whose max moved (PV_t(n-1) is complete: it was
      // issued before S_t(n), whose commit we waited on).
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_o + c * 32, o);
        }
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&bars->p_ready[t]);
    }
    if (ok && mbar_wait(&bars->o_final[t], 0, abort)) {
      tc_fence_after();
      const int h = h0 + t;
      const bool valid = i <= sc.q_hi;
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = p.out + ((static_cast<int64_t>(seq0) + i) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv, __uint_as_float(o[8 * v4 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv, __uint_as_float(o[8 * v4 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv, __uint_as_float(o[8 * v4 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv, __uint_as_float(o[8 * v4 + 7]) * inv);
            dst[v4] = w;
          }
        }
      }
      if (valid && p.lse != nullptr) {
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        p.lse[static_cast<int64_t>(h) * p.total_tokens + seq0 + i] = (m_use + log2f(l_run)) * 0.69314718055994531f;
      }
    }
  }

  // ---- teardown: every role is done; TMEM is released by its allocator warp ----
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

}  // namespace jl
