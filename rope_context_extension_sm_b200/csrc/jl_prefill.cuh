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
//   warp 1      TMEM allocator + tcgen05.mma issuer (warp-uniform loop, one
//               elected lane issues)
//   warps 2, 3  idle (the control warpgroup is complete for the register split)
//   warps 4..   one warpgroup per query head: the whole 128-column score row of
//               each thread read from TMEM once per tile, softmax in registers,
//               P written back to TMEM (bf16), O rescale, epilogue
//   last four   in-place RoPE rotation of the Q and K tiles in shared memory
//               (base rows R(x) or remote rows R(f(x))); each owns 32 rows and
//               steps its cos/sin factors along the rows by complex
//               multiplication with e^{i theta_c}, anchored once per tile on a
//               table row prefetched a tile ahead (no table load per row)
// Registers: launched at 65536 / threads per thread; setmaxnreg moves them from
// the control warpgroup (48) and the rotation warpgroup (80) to the softmax
// ones (192).
// TMEM columns: S_t at 128 t, O_t at 128 NQT + D t; P_t aliases S_t.
// With NQT = 2 the MMA issue order S0(n), PV1(n-1), S1(n), PV0(n) lets one
// head's softmax overlap the other head's tensor-core work.
#pragma once

#include "jl_device.cuh"

namespace jl {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kStages = 2;

// Optional timeline of one CTA (built only with -DJL_TRACE, for measurements):
// SM clock stamps of the roles' events on visits 100 .. 163 of CTA 0.
#ifdef JL_TRACE
__device__ long long g_trace[64 * 64];
#define JL_TRACE_AT(n, slot)                                                     \
  do {                                                                           \
    if (blockIdx.x == 0 && (n) >= 100 && (n) < 164 && (threadIdx.x & 31) == 0) \
      g_trace[((n) - 100) * 64 + (slot)] = clock64();                            \
  } while (0)
#else
#define JL_TRACE_AT(n, slot) \
  do {                       \
  } while (0)
#endif

struct PrefillParams {
  const int32_t* cu_seqlens;
  const float* cos_tab;
  const float* sin_tab;
  __nv_bfloat16* out;
  float* out_f32;        // if set, rows are written in fp32 here instead of bf16 to out
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
  int32_t mode;          // 0: fused bifocal / plain; 1: pass 1 alone; 3: pass 3 alone (see TileSchedule)
  int32_t cached;        // keys/values come from a base-RoPE cache (chunked prefill)
  // Keys arrive rotated (jl_key_rotate_kernel): rows [0, T) of the K map hold R(j) k_j for
  // local visits, rows [T, 2T) R(f(j)) k_j for remote visits; no K rotation in the kernel.
  int32_t krot;
  const float* cos_rem;  // frequency-interpolation variant: remote pairs rotate by these
  const float* sin_rem;  // rows at their raw positions (cos/sin(p theta_c lambda_c)); NULL = aliasing
  int64_t n_rem_rows;
  const int32_t* past_lens;  // cached: tokens in each cache entry before this chunk
  int64_t cache_stride;      // cached: positions per cache entry
  // Base-RoPE cache written by the prefill itself (NULL: not written): entry b, position j
  // gets R(j) k_j and v_j; [batch][cache_out_stride][Hkv][D].  v_raw is the packed V input.
  __nv_bfloat16* k_cache_out;
  __nv_bfloat16* v_cache_out;
  const __nv_bfloat16* v_raw;
  int64_t cache_out_stride;
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
  static constexpr int kRotWarps = 4;
  // Warpgroups: 0 = control (warp 0 TMA producer, warp 1 MMA issuer, warps 2-3
  // idle), 1 .. NQT = softmax (one per query head), NQT + 1 = rotation (warps
  // kR0 .. kR0 + 3).  Every warpgroup is complete, as the register split requires.
  static constexpr int kR0 = 4 + 4 * NQT;
  static constexpr int kWarps = kR0 + 4;
  static constexpr int kThreads = 32 * kWarps;
  // The softmax warpgroups hold a whole 128-column score row in registers and the
  // rotation warpgroup keeps eight rows of a tile in flight.  The block is
  // launched at kRegsLaunch registers per thread; the control warpgroup gives its
  // registers down to kRegsCtl and the rotation warpgroup to kRegsRot, the
  // softmax warpgroups take kRegsSoftmax.  Two heads: 128 x (48 + 2 x 192 + 80) =
  // 512 x 128, the whole register file.
  static constexpr bool kSplitRegs = true;
  static constexpr uint32_t kRegsLaunch = (65536 / kThreads) & ~7u;
  static constexpr uint32_t kRegsSoftmax = 192, kRegsCtl = 48, kRegsRot = 80;
  static constexpr uint32_t kRegsNeeded = 128 * (NQT * kRegsSoftmax + kRegsCtl + kRegsRot);
  static_assert(kRegsNeeded <= kThreads * kRegsLaunch, "register split exceeds the launch allocation");
  static_assert(kRegsRot <= kRegsLaunch && kRegsCtl <= kRegsLaunch, "a decrease must not exceed the launch count");
  __device__ static bool softmax_warp(int warp) { return warp >= 4 && warp < kR0; }
  __device__ static int rot_index(int warp) { return (warp >= kR0 && warp < kR0 + 4) ? warp - kR0 : -1; }
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

// Which key tiles a query block visits and in which order.  The fused kernel
// (visit_remote) visits remote tiles first, then local tiles.  The literal
// passes 1 and 3 of the inclusion-exclusion merge visit local tiles only (pass 2
// is the fused kernel with w0 = 0).
struct TileSchedule {
  int q_lo, q_hi;  // first / last valid query position of the block
  int n_kt;        // key tiles 0 .. n_kt-1 hold causal pairs
  int R;           // tiles holding a pair with i - j >= w0: kt in [0, R)
  int Lo;          // tiles holding a pair with i - j <  w0: kt in [Lo, n_kt)
  int n_virt;      // number of visits
  int w0;          // effective window (huge when every pair is local)
  bool visit_remote;

  __device__ void init(int q_first, int L, int w0_eff, bool with_remote) {
    w0 = w0_eff;
    visit_remote = with_remote;
    q_lo = q_first;
    q_hi = min(q_lo + kBM - 1, L - 1);
    n_kt = q_hi / kBN + 1;
    R = (q_hi >= w0) ? min(n_kt, (q_hi - w0) / kBN + 1) : 0;
    if (w0 <= 0) {
      Lo = n_kt;
    } else {
      const int x = q_lo - (kBN - 1) - w0;  // local iff kt * 128 > x
      Lo = (x < 0) ? 0 : min(n_kt, x / kBN + 1);
    }
    n_virt = (visit_remote ? R : 0) + (n_kt - Lo);
  }
  __device__ int R_visits() const { return visit_remote ? R : 0; }
  __device__ bool remote(int n) const { return n < R_visits(); }
  __device__ int kt(int n) const { return n < R_visits() ? n : Lo + (n - R_visits()); }
  // first visit of a Q rotation phase (remote phase, then local phase)
  __device__ bool phase_start(int n) const { return n == 0 || n == R_visits(); }
  // last visit using the remote-rotated Q when a local phase follows
  __device__ bool phase_end(int n) const { return n == R_visits() - 1 && R_visits() < n_virt; }
  // Does visit n need a per-element mask (window edge or causal diagonal)?
  __device__ bool masked(int n) const {
    const int k = kt(n);
    const bool diag = k * kBN + kBN - 1 > q_lo;
    return diag || (remote(n) ? (k >= Lo) : (k < R));
  }
};

// cos/sin of the frequencies a lane owns: c = 2l, 2l+1 (D = 128) or c = l (D = 64);
// each is paired with channel c + D/2 (rotate-half).
template <int D>
struct RotFactor {
  static constexpr int NF = D / 64;
  float c[NF], s[NF];
};

// Factor of table row `row` (base table, or the interpolated remote table when rem).
template <int D>
__device__ __forceinline__ void load_factor(RotFactor<D>& f, const PrefillParams& p, int64_t row, int lane,
                                            bool rem = false) {
  const float* ct = rem ? p.cos_rem : p.cos_tab;
  const float* st = rem ? p.sin_rem : p.sin_tab;
  const int64_t max_row = (rem ? p.n_rem_rows : p.n_tab_rows) - 1;
  row = row > max_row ? max_row : row;  // only rows past every sequence end are clamped
  if constexpr (D == 128) {
    const float2 cc = ldg_now_f2(ct + row * 64 + 2 * lane);
    const float2 ss = ldg_now_f2(st + row * 64 + 2 * lane);
    f.c[0] = cc.x; f.c[1] = cc.y; f.s[0] = ss.x; f.s[1] = ss.y;
  } else {
    f.c[0] = ldg_now_f(ct + row * 32 + lane);
    f.s[0] = ldg_now_f(st + row * 32 + lane);
  }
}

// f <- f * e^{i theta}: R(m) -> R(m + 1).
template <int D>
__device__ __forceinline__ void advance(RotFactor<D>& f, const RotFactor<D>& st) {
#pragma unroll
  for (int i = 0; i < RotFactor<D>::NF; ++i) {
    const float c = f.c[i] * st.c[i] - f.s[i] * st.s[i];
    const float sn = f.s[i] * st.c[i] + f.c[i] * st.s[i];
    f.c[i] = c;
    f.s[i] = sn;
  }
}

// Rotate row r of a 128-byte-swizzled [128 rows][D] bf16 tile in place with factor
// f = (cos, sin)(m theta): by R(m), or by R(-m) when INV.
template <int D, bool INV = false>
__device__ __forceinline__ void rotate_row(uint8_t* tile, int r, const RotFactor<D>& f, int lane) {
  constexpr float sg = INV ? -1.f : 1.f;
  if constexpr (D == 128) {
    // elements 2l, 2l+1 (box 0) and 64+2l, 64+2l+1 (box 1) share the swizzled offset
    const int off = r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + ((lane & 3) << 2);
    uint32_t* plo = reinterpret_cast<uint32_t*>(tile + off);
    uint32_t* phi = reinterpret_cast<uint32_t*>(tile + 16384 + off);
    const float2 a = unpack_bf16x2(*plo);
    const float2 b = unpack_bf16x2(*phi);
    // ya = a c - b s, yb = b c + a s on packed pairs (two frequencies per instruction)
    const uint64_t c2 = f2_pack(f.c[0], f.c[1]);
    const uint64_t s2 = f2_pack(sg * f.s[0], sg * f.s[1]);
    const uint64_t ns2 = f2_pack(-sg * f.s[0], -sg * f.s[1]);
    const uint64_t a2 = f2_pack(a.x, a.y), b2 = f2_pack(b.x, b.y);
    float2 ya, yb;
    f2_unpack(f2_fma(b2, ns2, f2_mul(a2, c2)), ya.x, ya.y);
    f2_unpack(f2_fma(a2, s2, f2_mul(b2, c2)), yb.x, yb.y);
    *plo = pack_bf16x2(ya.x, ya.y);
    *phi = pack_bf16x2(yb.x, yb.y);
  } else {
    // D == 64: elements l and l + 32 of the single box
    const int c0 = lane, c1 = lane + 32;
    const int off0 = r * 128 + ((((c0 * 2) >> 4) ^ (r & 7)) << 4) + ((c0 * 2) & 15);
    const int off1 = r * 128 + ((((c1 * 2) >> 4) ^ (r & 7)) << 4) + ((c1 * 2) & 15);
    __nv_bfloat16* pa = reinterpret_cast<__nv_bfloat16*>(tile + off0);
    __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(tile + off1);
    const float a = __bfloat162float(*pa), b = __bfloat162float(*pb);
    const float sn = sg * f.s[0];
    *pa = __float2bfloat16_rn(a * f.c[0] - b * sn);
    *pb = __float2bfloat16_rn(b * f.c[0] + a * sn);
  }
}

// Table row of the first row of rotation slice rw (rows slices of `rows` rows):
// position base + rows rw, or its remote position floor(./G) (g = 1 selects base
// positions).
__device__ __forceinline__ int64_t slice_anchor_row(int base, int rw, int g, int rows = 32) {
  const int pos = base + rows * rw;
  return g == 1 ? pos : pos / g;
}

// Rotate rows [ROWS rw, ROWS rw + ROWS) of a tile whose row r sits at position base + r:
// by R(pos) when g == 1, by R(floor(pos / g)) otherwise.  f is the factor of the
// slice's first row; the (remote) position steps up every g rows.  When base is a
// multiple of 32, slices start on a group boundary for GS = g in {1, 2, 4} and the
// step rows are known at compile time; GS = 0 handles any g and any base with a
// running counter and selects.
template <int D, int GS, int ROWS = 32>
__device__ __forceinline__ void rotate_slice(uint8_t* tile, int rw, int base, int g, RotFactor<D> f,
                                             const RotFactor<D>& st, int lane) {
  uint8_t* slice = tile + ROWS * rw * 128;  // ROWS rows x 128 B; row & 7 == r & 7
  if constexpr (GS > 0) {
#pragma unroll 8
    for (int r = 0; r < ROWS; ++r) {
      rotate_row<D>(slice, r, f, lane);
      if ((r + 1) % GS == 0) advance<D>(f, st);
    }
  } else {
    int cnt = (base + ROWS * rw) % g;
#pragma unroll 8
    for (int r = 0; r < ROWS; ++r) {
      rotate_row<D>(slice, r, f, lane);
      cnt = (cnt + 1 == g) ? 0 : cnt + 1;
      RotFactor<D> nf = f;
      advance<D>(nf, st);
#pragma unroll
      for (int e = 0; e < RotFactor<D>::NF; ++e) {
        f.c[e] = cnt == 0 ? nf.c[e] : f.c[e];
        f.s[e] = cnt == 0 ? nf.s[e] : f.s[e];
      }
    }
  }
}

// head_dim 128: rows [ROWS rw, ROWS rw + ROWS) in batches of eight rows -- every
// load of a batch first, then the arithmetic, then the stores -- so eight rows'
// shared-memory loads are in flight together instead of one row at a time.  Row
// r = 8 k + e of the slice has r & 7 == e, so its swizzled offset is known at
// compile time up to the lane.  f steps by st every g rows (GS > 0: g == GS).
template <int GS, int ROWS = 32>
__device__ __forceinline__ void rotate_slice_b8(uint8_t* tile, int rw, int base, int g, RotFactor<128> f,
                                                const RotFactor<128>& st, int lane) {
  uint8_t* slice = tile + ROWS * rw * 128;
  int cnt = GS > 0 ? 0 : (base + ROWS * rw) % g;
#pragma unroll 1
  for (int r0 = 0; r0 < ROWS; r0 += 8) {
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int off = (r0 + e) * 128 + (((lane >> 2) ^ e) << 4) + ((lane & 3) << 2);
      lo[e] = *reinterpret_cast<const uint32_t*>(slice + off);
      hi[e] = *reinterpret_cast<const uint32_t*>(slice + 16384 + off);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 a = unpack_bf16x2(lo[e]);
      const float2 b = unpack_bf16x2(hi[e]);
      const uint64_t c2 = f2_pack(f.c[0], f.c[1]);
      const uint64_t s2 = f2_pack(f.s[0], f.s[1]), ns2 = f2_pack(-f.s[0], -f.s[1]);
      const uint64_t a2 = f2_pack(a.x, a.y), b2 = f2_pack(b.x, b.y);
      float2 ya, yb;
      f2_unpack(f2_fma(b2, ns2, f2_mul(a2, c2)), ya.x, ya.y);
      f2_unpack(f2_fma(a2, s2, f2_mul(b2, c2)), yb.x, yb.y);
      lo[e] = pack_bf16x2(ya.x, ya.y);
      hi[e] = pack_bf16x2(yb.x, yb.y);
      if constexpr (GS > 0) {
        if ((e + 1) % GS == 0) advance<128>(f, st);
      } else {
        cnt = (cnt + 1 == g) ? 0 : cnt + 1;
        RotFactor<128> nf = f;
        advance<128>(nf, st);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          f.c[q] = cnt == 0 ? nf.c[q] : f.c[q];
          f.s[q] = cnt == 0 ? nf.s[q] : f.s[q];
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int off = (r0 + e) * 128 + (((lane >> 2) ^ e) << 4) + ((lane & 3) << 2);
      *reinterpret_cast<uint32_t*>(slice + off) = lo[e];
      *reinterpret_cast<uint32_t*>(slice + 16384 + off) = hi[e];
    }
  }
}


template <int D, int ROWS = 32>
__device__ __forceinline__ void rotate_slice_any(uint8_t* tile, int rw, int base, int g, const RotFactor<D>& f,
                                                 const RotFactor<D>& st, int lane) {
  if constexpr (D == 128) {
    if ((base & 31) != 0) {
      rotate_slice_b8<0, ROWS>(tile, rw, base, g, f, st, lane);
      return;
    }
    switch (g) {
      case 1: rotate_slice_b8<1, ROWS>(tile, rw, base, g, f, st, lane); break;
      case 2: rotate_slice_b8<2, ROWS>(tile, rw, base, g, f, st, lane); break;
      case 4: rotate_slice_b8<4, ROWS>(tile, rw, base, g, f, st, lane); break;
      default: rotate_slice_b8<0, ROWS>(tile, rw, base, g, f, st, lane); break;
    }
    return;
  }
  if ((base & 31) != 0) {  // a chunk's query block need not start on a multiple of 32
    rotate_slice<D, 0, ROWS>(tile, rw, base, g, f, st, lane);
    return;
  }
  switch (g) {
    case 1: rotate_slice<D, 1, ROWS>(tile, rw, base, g, f, st, lane); break;
    case 2: rotate_slice<D, 2, ROWS>(tile, rw, base, g, f, st, lane); break;
    case 4: rotate_slice<D, 4, ROWS>(tile, rw, base, g, f, st, lane); break;
    default: rotate_slice<D, 0, ROWS>(tile, rw, base, g, f, st, lane); break;
  }
}

// Correct rows [ROWS rw, ROWS rw + ROWS) of a cached (base-RoPE) key tile at positions
// kbase + r to their remote rotation: R(f(j) - j) = R(-n_j), n_j = j - floor(j/G).
// n steps by one per row except where f steps up; kbase is a multiple of 128, so
// for G in {2, 4} those rows are compile-time.  f holds (cos, sin)(n theta) of the
// slice's first row.
template <int D, int GS, int ROWS = 32>
__device__ __forceinline__ void correct_slice(uint8_t* tile, int rw, int kbase, int G, RotFactor<D> f,
                                              const RotFactor<D>& st, int lane) {
  uint8_t* slice = tile + ROWS * rw * 128;
  if constexpr (GS > 0) {
#pragma unroll 8
    for (int r = 0; r < ROWS; ++r) {
      rotate_row<D, true>(slice, r, f, lane);
      if ((r + 1) % GS != 0) advance<D>(f, st);
    }
  } else {
    int cnt = (kbase + ROWS * rw) % G;
#pragma unroll 8
    for (int r = 0; r < ROWS; ++r) {
      rotate_row<D, true>(slice, r, f, lane);
      cnt = (cnt + 1 == G) ? 0 : cnt + 1;
      RotFactor<D> nf = f;
      advance<D>(nf, st);
#pragma unroll
      for (int e = 0; e < RotFactor<D>::NF; ++e) {
        f.c[e] = cnt != 0 ? nf.c[e] : f.c[e];
        f.s[e] = cnt != 0 ? nf.s[e] : f.s[e];
      }
    }
  }
}

// Copy rows [ROWS rw, ROWS rw + ROWS) of a rotated 128-byte-swizzled K tile (shared
// memory) and the same rows of raw V (global) to the cache rows of positions
// pos0 + r of entry b, for r < n_valid.  16-byte chunks; consecutive lanes write
// consecutive chunks of a row (D = 128: two rows per pass, D = 64: four).
template <int D, int ROWS = 32>
__device__ __forceinline__ void write_cache_slice(const uint8_t* tile, int rw, const PrefillParams& p, int b,
                                                  int pos0, int n_valid, int64_t v_tok0, int hkv, int lane) {
  constexpr int kChunks = D / 8;          // 16-byte chunks per row
  constexpr int kRowsPerPass = 32 / kChunks;
  const int c = lane % kChunks;           // chunk of the row this lane copies
  const int box = c >> 3, j = c & 7;      // 64-channel box and chunk inside its 128-byte row
#pragma unroll 4
  for (int r0 = 0; r0 < ROWS; r0 += kRowsPerPass) {
    const int r = r0 + lane / kChunks;    // row within the slice
    const int row = ROWS * rw + r;        // row within the tile
    if (row >= n_valid) continue;
    JL_CHECK(pos0 + row < p.cache_out_stride && v_tok0 + row < p.total_tokens && b < p.batch);
    const uint4 kw = *reinterpret_cast<const uint4*>(tile + box * 16384 + row * 128 + ((j ^ (row & 7)) << 4));
    const int64_t dst = ((static_cast<int64_t>(b) * p.cache_out_stride + pos0 + row) * p.Hkv + hkv) * D + c * 8;
    const int64_t src = ((v_tok0 + row) * p.Hkv + hkv) * D + c * 8;
    *reinterpret_cast<uint4*>(p.k_cache_out + dst) = kw;
    *reinterpret_cast<uint4*>(p.v_cache_out + dst) = *reinterpret_cast<const uint4*>(p.v_raw + src);
  }
}

// 2^x for a pair of values on the FMA and integer pipes instead of the MUFU unit.
// Range reduction: the nearest integer n of x comes from adding 1.5 * 2^23 (whose
// low mantissa bits then hold n); f = x - n lies in [-1/2, 1/2]; 2^f is a degree-3
// polynomial fitted here for minimum relative error on that interval (at most
// 7.5e-5, far below the bf16 rounding P gets); 2^n is added into the exponent
// field.  x is clamped to >= -125 so the result stays a normal number.
__device__ __forceinline__ void exp2_poly_x2(uint64_t x, float& y0, float& y1) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t shift = f2_pack(12582912.f, 12582912.f);
  const uint64_t t = f2_add(xc, shift);
  const uint64_t fr = f2_sub(xc, f2_sub(t, shift));
  uint64_t pl = f2_fma(fr, f2_pack(0.05517160892486572f, 0.05517160892486572f),
                       f2_pack(0.2426111102104187f, 0.2426111102104187f));
  pl = f2_fma(pl, fr, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  pl = f2_fma(pl, fr, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  float t0, t1, q0, q1;
  f2_unpack(t, t0, t1);
  f2_unpack(pl, q0, q1);
  y0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// p = 2^(s * sl2 - m) over NC score columns (zero outside [keep_lo + 1,
// keep_hi] when MASK), packed to bf16 pairs; accumulates the two partial row
// sums.  Every POLY-th pair of exponentials (0: none) is computed by
// exp2_poly_x2 on the FMA pipe, the rest on the MUFU unit.  Straight-line code:
// no branch inside.
template <bool MASK, int NC, int POLY = 0>
__device__ __forceinline__ void softmax_chunk(const uint32_t (&sr)[NC], uint32_t (&pk)[NC / 2], int col0, float sl2,
                                              float neg_m, int keep_lo, int keep_hi, float& lsum, float& lsum2) {
  const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
  uint64_t acc = f2_pack(lsum, lsum2);
#pragma unroll
  for (int e = 0; e < NC / 2; ++e) {
    // (s0, s1) * scale - m in one packed FMA, two ex2, one packed add into the row sums
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), scale2, negm2);
    float p0, p1;
    if (POLY > 0 && e % (POLY > 0 ? POLY : 1) == POLY - 1) {
      exp2_poly_x2(x, p0, p1);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    if constexpr (MASK) {
      const int col = col0 + 2 * e;
      p0 = (col > keep_lo && col <= keep_hi) ? p0 : 0.f;
      p1 = (col + 1 > keep_lo && col + 1 <= keep_hi) ? p1 : 0.f;
    }
    acc = f2_add(acc, f2_pack(p0, p1));
    pk[e] = pack_bf16x2(p0, p1);
  }
  f2_unpack(acc, lsum, lsum2);
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

  // ---- work item: KV-head-major so the CTAs in flight share one head's K/V in
  // L2; within a head, heaviest query blocks first ----
  const int per_head = p.n_qtiles * p.batch * p.slots;
  const int hkv = static_cast<int>(blockIdx.x) / per_head;
  const int rem = static_cast<int>(blockIdx.x) % per_head;
  const int qt = p.n_qtiles - 1 - rem / (p.batch * p.slots);
  const int b = (rem / p.slots) % p.batch;
  const int slot = rem % p.slots;
  const int h0 = hkv * p.group + slot * NQT;
  const int seq0 = p.cu_seqlens[b];                 // packed index of the sequence's first query
  const int n_rows = p.cu_seqlens[b + 1] - seq0;    // queries of this sequence (or chunk)
  if (qt * kBM >= n_rows) return;  // uniform across the CTA, before any barrier exists
  if (status_failed()) return;
  const int past = p.cached ? p.past_lens[b] : 0;   // chunked prefill: keys already cached
  const int L = past + n_rows;                      // sequence length after this chunk
  const int q_tok0 = seq0 + qt * kBM;               // packed index of the block's first query

  const bool interp = p.cos_rem != nullptr;  // remote pairs: interpolated table, no aliasing
  int G = 1;
  if (!p.plain && !interp) G = max(1, (L + p.w_pre - 1) / p.w_pre);
  // G = 1 (or plain): remote scores equal base scores, every pair runs as local.
  // The literal passes keep the real window.
  const int w0_eff = (p.mode == 0 && !interp && (p.plain || G == 1)) ? (1 << 30) : p.w0;
  TileSchedule sc;
  sc.init(past + qt * kBM, L, w0_eff, p.mode == 0);
  // Pass 3 rotates its (local-window) visits by the remote positions.
  const bool local_uses_remote = (p.mode == 3);

  if (sc.n_virt == 0) {  // an empty pass (w0 = 0 for passes 1 and 3): O = 0, lse = -inf
    for (int r = threadIdx.x; r < kBM * NQT; r += blockDim.x) {
      const int i = sc.q_lo + (r % kBM), h = h0 + r / kBM;
      if (i > sc.q_hi) continue;
      const int64_t tok = q_tok0 + (r % kBM);
      const int64_t row_off = (tok * p.Hq + h) * D;
      for (int c = 0; c < D; ++c) {
        if (p.out_f32 != nullptr) p.out_f32[row_off + c] = 0.f;
        else p.out[row_off + c] = __float2bfloat16_rn(0.f);
      }
      if (p.lse != nullptr) p.lse[static_cast<int64_t>(h) * p.total_tokens + tok] = -INFINITY;
    }
    return;
  }

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
    mbar_init(&bars->q_ready, Lay::kRotWarps);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_ready[s], Lay::kRotWarps);
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
  // Register split: each role's first instruction, executed by the whole warp
  // (every warp of a warpgroup takes the same share).
  auto give_regs = [] {  // control warpgroup
    if constexpr (Lay::kSplitRegs) setmaxnreg_dec<Lay::kRegsCtl>();
  };

  if (warp == 0) {
    give_regs();
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued_q = 0;
      int issued[kStages] = {0};
      JL_CHECK(q_tok0 >= 0 && q_tok0 < p.total_tokens && h0 + NQT <= p.Hq && hkv < p.Hkv);
      for (int n = 0; n < sc.n_virt && !*abort; ++n) {
        if (sc.phase_start(n)) {
          if (n > 0 && !mbar_wait(&bars->q_empty, 0, abort)) break;
          mbar_arrive_expect_tx(&bars->q_full, kTileTx * NQT);
          for (int t = 0; t < NQT; ++t)
            for (int bx = 0; bx < NBOX; ++bx)
              tma_load_3d(sQ + t * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_q, &bars->q_full, bx * 64, h0 + t,
                          q_tok0);
          ++issued_q;
        }
        const int s = n % kStages;
        const uint32_t u = n / kStages;
        const int key0 = p.cached ? static_cast<int>(b * p.cache_stride) + sc.kt(n) * kBN : seq0 + sc.kt(n) * kBN;
        // the tile's causal keys lie inside this sequence's keys (packed prompt or cache entry)
        JL_CHECK(key0 >= 0 && sc.kt(n) * kBN < L &&
                 key0 + min(kBN - 1, L - 1 - sc.kt(n) * kBN) <
                     (p.cached ? static_cast<int64_t>(b) * p.cache_stride + (L < p.cache_stride ? L : p.cache_stride)
                               : static_cast<int64_t>(seq0) + n_rows));
        // pre-rotated keys: a remote visit reads the R(f(j)) k rows, T rows on
        const int krow = key0 + ((p.krot && sc.remote(n)) ? static_cast<int>(p.total_tokens) : 0);
        if (u > 0 && !mbar_wait(&bars->k_empty[s], (u - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], kTileTx);
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(sK + s * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_k, &bars->k_full[s], bx * 64, hkv, krow);
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
    give_regs();
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs the loop, so every operand stays warp-uniform; one
    // elected lane issues each tcgen05 instruction.  Descriptors are formed
    // once: the descriptor of (base + off) is that of base plus off / 16 (the
    // start-address field, which cannot carry below 256 KB of shared memory).
    const bool leader = elect_one();
    const uint64_t dq0 = sdesc_kmajor_sw128(smem_u32(sQ));
    const uint64_t dk0 = sdesc_kmajor_sw128(smem_u32(sK));
    const uint64_t dv0 = sdesc_mnmajor_sw128(smem_u32(sV), 16384);
    auto issue_s = [&](int t, int s) {
      const uint64_t qd = dq0 + static_cast<uint32_t>((t * Lay::kTileBytes) >> 4);
      const uint64_t kd = dk0 + static_cast<uint32_t>((s * Lay::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        constexpr uint32_t kBox16 = Lay::kBoxBytes >> 4;
        const uint32_t off = (kk >> 2) * kBox16 + (kk & 3) * 2;
        if (leader) umma_ss(tmem + t * 128, qd + off, kd + off, kIdescS, kk > 0);
      }
    };
    auto issue_pv = [&](int t, int s, bool acc) {
      const uint64_t vd = dv0 + static_cast<uint32_t>((s * Lay::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < PSTEPS; ++kk)
        if (leader)
          umma_ts(tmem + NQT * 128 + t * D, tmem + t * 128 + kk * 8, vd + kk * (2048 >> 4), kIdescO,
                  (acc || kk > 0) ? 1u : 0u);
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) umma_commit(bar);
    };
    int n = 0;
    bool ok = true;
    for (; n < sc.n_virt && ok; ++n) {
      if (sc.phase_start(n)) {
        if (!(ok = warp_wait(&bars->q_ready, n == 0 ? 0 : 1, abort))) break;
        tc_fence_after();
      }
      const int s = n % kStages;
      const uint32_t u = n / kStages;
      JL_TRACE_AT(n, 0);
      if (!(ok = warp_wait(&bars->k_ready[s], u & 1, abort))) break;
      JL_TRACE_AT(n, 1);
      tc_fence_after();
      issue_s(0, s);
      commit(&bars->s_full[0]);
      if (NQT == 2) {
        if (n > 0) {
          const int sp = (n - 1) % kStages;
          if (!(ok = warp_wait(&bars->p_ready[1], (n - 1) & 1, abort))) break;
          tc_fence_after();
          if (!(ok = warp_wait(&bars->v_full[sp], ((n - 1) / kStages) & 1, abort))) break;
          issue_pv(1, sp, n - 1 > 0);
          commit(&bars->v_empty[sp]);
        }
        issue_s(1, s);
        commit(&bars->s_full[1]);
        JL_TRACE_AT(n, 3);
      }
      commit(&bars->k_empty[s]);
      if (sc.phase_end(n)) commit(&bars->q_empty);
      JL_TRACE_AT(n, 2);
      if (!(ok = warp_wait(&bars->p_ready[0], n & 1, abort))) break;
      JL_TRACE_AT(n, 4);
      tc_fence_after();
      if (!(ok = warp_wait(&bars->v_full[s], u & 1, abort))) break;
      issue_pv(0, s, n > 0);
      if (NQT == 1) commit(&bars->v_empty[s]);
    }
    if (ok && NQT == 2) {
      const int nl = sc.n_virt - 1;
      const int sl = nl % kStages;
      ok = warp_wait(&bars->p_ready[1], nl & 1, abort);
      if (ok) {
        tc_fence_after();
        ok = warp_wait(&bars->v_full[sl], (nl / kStages) & 1, abort);
      }
      if (ok) {
        issue_pv(1, sl, nl > 0);
        commit(&bars->v_empty[sl]);
      }
    }
    if (ok) {
      commit(&bars->o_final[0]);
      if (NQT == 2) commit(&bars->o_final[1]);
    }
    // Every issued MMA must finish before TMEM is released.
    commit(&bars->teardown);
    mbar_wait_bounded(&bars->teardown, 0);
    __syncwarp();
  } else if (Lay::rot_index(warp) >= 0) {
    if constexpr (Lay::kSplitRegs) setmaxnreg_dec<Lay::kRegsRot>();
    // ------------------------------------------------------------ rotation
    const int rw = Lay::rot_index(warp);
    {
    RotFactor<D> step, step_rem;  // e^{i theta_c} (row 1 of the base table) and of the interpolated table
    load_factor<D>(step, p, 1, lane);
    if (interp) load_factor<D>(step_rem, p, 1, lane, true);
    // Table row of the slice's first key in visit m (called for m = 0, 1, 2, ... in
    // order): the quotient by G is stepped from the previous visit (the next key tile
    // is 128 positions on) and divided afresh only when the tile run or the divisor
    // changes, so the loop issues no integer division (see StepDiv).
    StepDiv kdiv{};
    int kdiv_kt = -2, kdiv_g = 0;
    auto key_anchor = [&](int m) -> int64_t {
      const int gm = p.cached ? G : ((sc.remote(m) || local_uses_remote) ? G : 1);
      const int pos = sc.kt(m) * kBN + 32 * rw;
      if (gm == 1) return p.cached ? 0 : pos;
      if (sc.kt(m) == kdiv_kt + 1 && gm == kdiv_g) kdiv.next();
      else kdiv.init(pos, kBN, gm);
      kdiv_kt = sc.kt(m);
      kdiv_g = gm;
      return p.cached ? pos - kdiv.q : kdiv.q;  // cached: correction index n_j = j - f(j)
    };
    RotFactor<D> fk_next;
    if (!p.krot) load_factor<D>(fk_next, p, key_anchor(0), lane, interp && sc.remote(0));
    const bool write_cache = p.k_cache_out != nullptr && slot == 0 && p.mode == 0 && !p.cached;
    for (int n = 0; n < sc.n_virt; ++n) {
      const bool remote = sc.remote(n);
      const bool rem_tab = interp && remote;  // interpolated rows at raw positions
      const int g = (!interp && (remote || local_uses_remote)) ? G : 1;
      const RotFactor<D>& stp = rem_tab ? step_rem : step;
      if (sc.phase_start(n)) {
        RotFactor<D> fq;
        load_factor<D>(fq, p, slice_anchor_row(sc.q_lo, rw, g), lane, rem_tab);
        {  // table rows of this slice's valid query rows
          const int first = sc.q_lo + 32 * rw, last = min(first + 31, L - 1);
          JL_CHECK(first > last || (last / g < (rem_tab ? p.n_rem_rows : p.n_tab_rows) &&
                                    (g == 1 || interp || last / g < p.w_pre)));
        }
        if (!mbar_wait(&bars->q_full, n == 0 ? 0 : 1, abort)) break;
        for (int t = 0; t < NQT; ++t) rotate_slice_any<D>(sQ + t * Lay::kTileBytes, rw, sc.q_lo, g, fq, stp, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_ready);
      }
      const RotFactor<D> fk = fk_next;
      if (n + 1 < sc.n_virt && !p.krot)  // prefetch a tile ahead
        load_factor<D>(fk_next, p, key_anchor(n + 1), lane, interp && sc.remote(n + 1));
      const int s = n % kStages;
      {  // table rows of this slice's valid keys: base R(j), remote R(j / G) (< w_pretrained), or the
         // cached keys' correction rows j - j / G
        const int first = sc.kt(n) * kBN + 32 * rw, last = min(first + 31, L - 1);
        if (p.cached)
          JL_CHECK(first > last || g == 1 || last - last / G < p.n_tab_rows);
        else
          JL_CHECK(first > last || (last / g < (rem_tab ? p.n_rem_rows : p.n_tab_rows) &&
                                    (g == 1 || interp || last / g < p.w_pre)));
      }
      JL_TRACE_AT(n, 5 + 3 * rw);
      if (!mbar_wait(&bars->k_full[s], (n / kStages) & 1, abort)) break;
      JL_TRACE_AT(n, 6 + 3 * rw);
      if (p.krot) {
        // the keys arrived rotated for this visit's kind
      } else if (!p.cached) {
        rotate_slice_any<D>(sK + s * Lay::kTileBytes, rw, sc.kt(n) * kBN, g, fk, stp, lane);
        // The query block's own key tile, visited as local, now holds R(j) k_j: the first
        // head slot of the KV group writes it (and the raw V rows) to the cache before the
        // tile is released to the MMA, whose commit frees the stage.
        if (write_cache && !remote && sc.kt(n) == qt) {
          __syncwarp();
          write_cache_slice<D>(sK + s * Lay::kTileBytes, rw, p, b, qt * kBN, n_rows - qt * kBN, q_tok0, hkv, lane);
        }
      } else if (g > 1) {  // cached keys are base-rotated: local visits use them as they are
        switch (g) {
          case 2: correct_slice<D, 2>(sK + s * Lay::kTileBytes, rw, sc.kt(n) * kBN, g, fk, step, lane); break;
          case 4: correct_slice<D, 4>(sK + s * Lay::kTileBytes, rw, sc.kt(n) * kBN, g, fk, step, lane); break;
          default: correct_slice<D, 0>(sK + s * Lay::kTileBytes, rw, sc.kt(n) * kBN, g, fk, step, lane); break;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->k_ready[s]);
      JL_TRACE_AT(n, 7 + 3 * rw);
    }
    }
  } else if (Lay::softmax_warp(warp)) {
    if constexpr (Lay::kSplitRegs) setmaxnreg_inc<Lay::kRegsSoftmax>();
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
      JL_TRACE_AT(n, 20 + 20 * t + 5 * wq);
      tc_fence_after();
      // The whole score row in registers: one TMEM round trip per tile.
      uint32_t sr[128];
      tmem_ld128(t_s, sr);
      const bool msk = sc.masked(n);
      const int hi = i - sc.kt(n) * kBN;  // causal: keep column c <= hi
      const int edge = hi - sc.w0;        // remote keeps c <= edge, local keeps c > edge
      const bool rem = sc.remote(n);
      const int keep_lo = msk ? (rem ? -1 : edge) : -1;     // keep c > keep_lo
      const int keep_hi = msk ? (rem ? edge : hi) : kBN;    // keep c <= keep_hi
      float mx = -INFINITY;
      if (msk) {
#pragma unroll
        for (int e = 0; e < 128; ++e) mx = (e > keep_lo && e <= keep_hi) ? fmaxf(mx, __uint_as_float(sr[e])) : mx;
      } else {
        float m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; e += 8) {
          mx = fmax3(mx, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
          m1 = fmax3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
          m2 = fmax3(m2, __uint_as_float(sr[e + 4]), __uint_as_float(sr[e + 5]));
          m3 = fmax3(m3, __uint_as_float(sr[e + 6]), __uint_as_float(sr[e + 7]));
        }
        mx = fmaxf(fmaxf(mx, m1), fmaxf(m2, m3));
      }
      const float m_new = fmaxf(m_run, mx * sl2);
      // Lazy rescale: keep the stale max unless the new one exceeds it by > 8 (x256).
      const bool resc = (m_run != -INFINITY) && (m_new > m_run + 8.f);
      const float alpha = resc ? ex2_approx(m_run - m_new) : 1.f;
      if (resc || m_run == -INFINITY) m_run = m_new;
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      JL_TRACE_AT(n, 21 + 20 * t + 5 * wq);
      JL_TRACE_AT(n, 22 + 20 * t + 5 * wq);
      // P = 2^(s * scale_log2 - m) as bf16 pairs over S columns [0, 64).
      float lsum = 0.f, lsum2 = 0.f;
      uint32_t pk[64];
      if (msk) softmax_chunk<true, 128>(sr, pk, 0, sl2, -m_use, keep_lo, keep_hi, lsum, lsum2);
      else softmax_chunk<false, 128>(sr, pk, 0, sl2, -m_use, keep_lo, keep_hi, lsum, lsum2);
      lsum += lsum2;
      JL_TRACE_AT(n, 23 + 20 * t + 5 * wq);
      tmem_st64(t_s, pk);
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
      JL_TRACE_AT(n, 24 + 20 * t + 5 * wq);
    }
    if (ok && mbar_wait(&bars->o_final[t], 0, abort)) {
      tc_fence_after();
      const int h = h0 + t;
      const bool valid = i <= sc.q_hi;
      JL_CHECK(!valid || (static_cast<int64_t>(q_tok0) + row < p.total_tokens && h < p.Hq));
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const int64_t row_off = ((static_cast<int64_t>(q_tok0) + row) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        if (valid && p.out_f32 != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.out_f32 + row_off + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(o[4 * v4]) * inv, __uint_as_float(o[4 * v4 + 1]) * inv,
                                  __uint_as_float(o[4 * v4 + 2]) * inv, __uint_as_float(o[4 * v4 + 3]) * inv);
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + row_off + c * 32);
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
        p.lse[static_cast<int64_t>(h) * p.total_tokens + q_tok0 + row] = (m_use + log2f(l_run)) * 0.69314718055994531f;
      }
    }
  }

  if (warp == 2 || warp == 3) give_regs();  // the control warpgroup's idle warps still give their share

  // ---- teardown: every role is done; TMEM is released by its allocator warp ----
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

// head_dim 128, 16-row slices, 16-byte shared-memory accesses.  Lane l owns the
// eight frequencies 8 c .. 8 c + 7 (c = l & 7): one 16-byte chunk of box 0 and the
// same chunk of box 1; lane group q = l >> 3 takes rows 4 q .. 4 q + 3 of the slice
// in order, so one warp instruction moves four rows and a slice takes a quarter of
// the shared-memory instructions of the 4-byte form (those share the issue queue
// with the MUFU unit the softmax runs on).  All four rows are loaded before any is
// computed.  f = (cos, sin) of the lane's frequencies at its first row, stepped by
// st every g rows (GS > 0: g == GS).
struct RotFactor8 {
  float c[8], s[8];
};

__device__ __forceinline__ void load_factor8(RotFactor8& f, const float* ct, const float* stb, int64_t row,
                                             int64_t max_row, int c8) {
  row = row > max_row ? max_row : row;
  const float4* pc = reinterpret_cast<const float4*>(ct + row * 64 + 8 * c8);
  const float4* ps = reinterpret_cast<const float4*>(stb + row * 64 + 8 * c8);
  const float4 c0 = pc[0], c1 = pc[1], s0 = ps[0], s1 = ps[1];
  f.c[0] = c0.x; f.c[1] = c0.y; f.c[2] = c0.z; f.c[3] = c0.w; f.c[4] = c1.x; f.c[5] = c1.y; f.c[6] = c1.z; f.c[7] = c1.w;
  f.s[0] = s0.x; f.s[1] = s0.y; f.s[2] = s0.z; f.s[3] = s0.w; f.s[4] = s1.x; f.s[5] = s1.y; f.s[6] = s1.z; f.s[7] = s1.w;
}

__device__ __forceinline__ void advance8(RotFactor8& f, const RotFactor8& st) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const uint64_t c2 = f2_pack(f.c[i], f.c[i + 1]), s2 = f2_pack(f.s[i], f.s[i + 1]);
    const uint64_t tc = f2_pack(st.c[i], st.c[i + 1]), ts = f2_pack(st.s[i], st.s[i + 1]);
    const uint64_t nc = f2_fma(c2, tc, f2_mul(f2_pack(-f.s[i], -f.s[i + 1]), ts));
    const uint64_t ns = f2_fma(s2, tc, f2_mul(c2, ts));
    f2_unpack(nc, f.c[i], f.c[i + 1]);
    f2_unpack(ns, f.s[i], f.s[i + 1]);
  }
}

template <int GS>
__device__ __forceinline__ void rotate_slice_v128(uint8_t* tile, int rw, int cnt0, int g, RotFactor8 f,
                                                  const RotFactor8& st, int lane) {
  const int c8 = lane & 7, row0 = 16 * rw + 4 * (lane >> 3);
  int cnt = cnt0;  // (position of the lane's first row) mod g, for the general path
  uint4 lo[4], hi[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int r = row0 + e;
    const int off = r * 128 + ((c8 ^ (r & 7)) << 4);
    lo[e] = *reinterpret_cast<const uint4*>(tile + off);
    hi[e] = *reinterpret_cast<const uint4*>(tile + 16384 + off);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t wl[4] = {lo[e].x, lo[e].y, lo[e].z, lo[e].w}, wh[4] = {hi[e].x, hi[e].y, hi[e].z, hi[e].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {  // frequencies 2 w, 2 w + 1 of the lane's eight
      const float2 a = unpack_bf16x2(wl[w]);
      const float2 b = unpack_bf16x2(wh[w]);
      const uint64_t c2 = f2_pack(f.c[2 * w], f.c[2 * w + 1]);
      const uint64_t s2 = f2_pack(f.s[2 * w], f.s[2 * w + 1]), ns2 = f2_pack(-f.s[2 * w], -f.s[2 * w + 1]);
      const uint64_t a2 = f2_pack(a.x, a.y), b2 = f2_pack(b.x, b.y);
      float2 ya, yb;
      f2_unpack(f2_fma(b2, ns2, f2_mul(a2, c2)), ya.x, ya.y);
      f2_unpack(f2_fma(a2, s2, f2_mul(b2, c2)), yb.x, yb.y);
      wl[w] = pack_bf16x2(ya.x, ya.y);
      wh[w] = pack_bf16x2(yb.x, yb.y);
    }
    lo[e] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    hi[e] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    if constexpr (GS > 0) {
      if ((e + 1) % GS == 0) advance8(f, st);
    } else {
      cnt = (cnt + 1 == g) ? 0 : cnt + 1;
      RotFactor8 nf = f;
      advance8(nf, st);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        f.c[q] = cnt == 0 ? nf.c[q] : f.c[q];
        f.s[q] = cnt == 0 ? nf.s[q] : f.s[q];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int r = row0 + e;
    const int off = r * 128 + ((c8 ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(tile + off) = lo[e];
    *reinterpret_cast<uint4*>(tile + 16384 + off) = hi[e];
  }
}

// base: position of the tile's first row; cnt0: (position of this lane's first
// row) mod g (unused when g is 1, 2 or 4 and base a multiple of 4).
__device__ __forceinline__ void rotate_slice_v128_any(uint8_t* tile, int rw, int base, int cnt0, int g,
                                                      const RotFactor8& f, const RotFactor8& st, int lane) {
  if ((base & 3) != 0) {  // a chunk's query block need not start on a multiple of 4
    rotate_slice_v128<0>(tile, rw, cnt0, g, f, st, lane);
    return;
  }
  switch (g) {
    case 1: rotate_slice_v128<1>(tile, rw, 0, g, f, st, lane); break;
    case 2: rotate_slice_v128<2>(tile, rw, 0, g, f, st, lane); break;
    case 4: rotate_slice_v128<4>(tile, rw, 0, g, f, st, lane); break;
    default: rotate_slice_v128<0>(tile, rw, cnt0, g, f, st, lane); break;
  }
}

// ===================================================== one head per CTA, S double-buffered
//
// The same computation as jl_prefill_kernel with one query head per CTA and two S
// buffers in TMEM (S0 at column 0, S1 at 128, O at 256).  The MMA warp issues
// S(n + 2) into buffer n & 1 right after PV(n) has read P(n) there (one issuer, the
// tensor pipe runs its MMAs in order), so the scores of the next tile are ready
// while the softmax of this one runs: the softmax warpgroup goes from tile to tile
// without waiting for PV(n) -> S(n + 1), and it has the MUFU unit to itself.  Eight
// rotation warps (16 rows each) rotate every K tile for this one head.  K takes three
// stages and V two, each with its own producer warp.
//   warp 0      TMA producer of Q and K
//   warp 1      TMEM allocator + tcgen05.mma issuer (warp-uniform, one elected lane)
//   warp 2      TMA producer of V
//   warp 3      idle (the control warpgroup is complete for the register split)
//   warps 4-7   softmax + O rescale + epilogue (thread = query row)
//   warps 8-15  RoPE rotation of the Q and K tiles in shared memory
// Every JL_DB_POLY-th pair of a score row's exponentials runs on the FMA pipe
// (0: all on the MUFU unit).
#ifndef JL_DB_POLY
#define JL_DB_POLY 0
#endif

template <int D>
struct PrefillDbLayout {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kBar = kV + kVStages * kTileBytes;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;  // S0, S1, O
  static constexpr int kOCol = 256;
  static constexpr int kRotWarps = 8;
  static constexpr int kRotRows = kBM / kRotWarps;  // 16
  static constexpr int kWarps = 16;
  static constexpr int kThreads = 32 * kWarps;
  // Launched at 128 registers per thread; the control warpgroup gives its
  // registers down to kRegsCtl, the two rotation warpgroups to kRegsRot, the
  // softmax warpgroup takes kRegsSoftmax: 128 x (48 + 224 + 2 x 120) = 512 x 128.
  static constexpr uint32_t kRegsLaunch = 65536 / kThreads;
  static constexpr uint32_t kRegsSoftmax = 224, kRegsCtl = 48, kRegsRot = 120;
  static constexpr uint32_t kRegsNeeded = 128 * (kRegsSoftmax + kRegsCtl + 2 * kRegsRot);
  static_assert(kRegsNeeded <= kThreads * kRegsLaunch, "register split exceeds the launch allocation");
  static_assert(kRegsRot <= kRegsLaunch && kRegsCtl <= kRegsLaunch, "a decrease must not exceed the launch count");
  static_assert(kBytes <= 232448 - 1024, "shared memory");
};

struct PrefillDbBars {
  uint64_t q_full, q_ready, q_empty;
  uint64_t k_full[3], k_ready[3], k_empty[3];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], p_ready[2], pv_done, o_final;
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(PrefillDbLayout<D>::kThreads, 1)
    jl_prefill_db_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using Lay = PrefillDbLayout<D>;
  constexpr int NBOX = D / 64;
  constexpr uint32_t kTileTx = kBM * D * 2;
  constexpr int KSTEPS = D / 16;
  constexpr int PSTEPS = kBN / 16;
  constexpr int RR = Lay::kRotRows;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, false, true);

  // ---- work item (KV-head-major, heaviest query blocks first; one head) ----
  const int per_head = p.n_qtiles * p.batch * p.slots;
  const int hkv = static_cast<int>(blockIdx.x) / per_head;
  const int rem = static_cast<int>(blockIdx.x) % per_head;
  const int qt = p.n_qtiles - 1 - rem / (p.batch * p.slots);
  const int b = (rem / p.slots) % p.batch;
  const int slot = rem % p.slots;
  const int h = hkv * p.group + slot;
  const int seq0 = p.cu_seqlens[b];
  const int n_rows = p.cu_seqlens[b + 1] - seq0;
  if (qt * kBM >= n_rows) return;
  if (status_failed()) return;
  const int past = p.cached ? p.past_lens[b] : 0;
  const int L = past + n_rows;
  const int q_tok0 = seq0 + qt * kBM;

  const bool interp = p.cos_rem != nullptr;
  int G = 1;
  if (!p.plain && !interp) G = max(1, (L + p.w_pre - 1) / p.w_pre);
  const int w0_eff = (p.mode == 0 && !interp && (p.plain || G == 1)) ? (1 << 30) : p.w0;
  TileSchedule sc;
  sc.init(past + qt * kBM, L, w0_eff, p.mode == 0);
  const bool local_uses_remote = (p.mode == 3);

  if (sc.n_virt == 0) {  // an empty pass: O = 0, lse = -inf
    for (int r = threadIdx.x; r < kBM; r += blockDim.x) {
      const int i = sc.q_lo + r;
      if (i > sc.q_hi) continue;
      const int64_t tok = q_tok0 + r;
      const int64_t row_off = (tok * p.Hq + h) * D;
      for (int c = 0; c < D; ++c) {
        if (p.out_f32 != nullptr) p.out_f32[row_off + c] = 0.f;
        else p.out[row_off + c] = __float2bfloat16_rn(0.f);
      }
      if (p.lse != nullptr) p.lse[static_cast<int64_t>(h) * p.total_tokens + tok] = -INFINITY;
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem + Lay::kQ;
  uint8_t* sK = smem + Lay::kK;
  uint8_t* sV = smem + Lay::kV;
  PrefillDbBars* bars = reinterpret_cast<PrefillDbBars*>(smem + Lay::kBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_ready, Lay::kRotWarps);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < Lay::kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_ready[s], Lay::kRotWarps);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < Lay::kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_ready[t], 128);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_final, 1);
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
  auto give_regs = [] { setmaxnreg_dec<Lay::kRegsCtl>(); };

  if (warp == 0) {
    give_regs();
    // ------------------------------------------------------ Q and K producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      int issued_q = 0;
      int issued[Lay::kKStages] = {0};
      JL_CHECK(q_tok0 >= 0 && q_tok0 < p.total_tokens && h < p.Hq && hkv < p.Hkv);
      for (int n = 0; n < sc.n_virt && !*abort; ++n) {
        if (sc.phase_start(n)) {
          if (n > 0 && !mbar_wait(&bars->q_empty, 0, abort)) break;
          mbar_arrive_expect_tx(&bars->q_full, kTileTx);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(sQ + bx * Lay::kBoxBytes, &tm_q, &bars->q_full, bx * 64, h, q_tok0);
          ++issued_q;
        }
        const int s = n % Lay::kKStages;
        const uint32_t u = n / Lay::kKStages;
        const int key0 = p.cached ? static_cast<int>(b * p.cache_stride) + sc.kt(n) * kBN : seq0 + sc.kt(n) * kBN;
        JL_CHECK(key0 >= 0 && sc.kt(n) * kBN < L &&
                 key0 + min(kBN - 1, L - 1 - sc.kt(n) * kBN) <
                     (p.cached ? static_cast<int64_t>(b) * p.cache_stride + (L < p.cache_stride ? L : p.cache_stride)
                               : static_cast<int64_t>(seq0) + n_rows));
        // pre-rotated keys: a remote visit reads the R(f(j)) k rows, T rows on
        const int krow = key0 + ((p.krot && sc.remote(n)) ? static_cast<int>(p.total_tokens) : 0);
        if (u > 0 && !mbar_wait(&bars->k_empty[s], (u - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], kTileTx);
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(sK + s * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_k, &bars->k_full[s], bx * 64, hkv, krow);
        issued[s] = static_cast<int>(u) + 1;
      }
      if (issued_q > 0) mbar_wait_bounded(&bars->q_full, (issued_q - 1) & 1);
      for (int s = 0; s < Lay::kKStages; ++s)
        if (issued[s] > 0) mbar_wait_bounded(&bars->k_full[s], (issued[s] - 1) & 1);
    }
  } else if (warp == 2) {
    give_regs();
    // ----------------------------------------------------------- V producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      int issued[Lay::kVStages] = {0};
      for (int n = 0; n < sc.n_virt && !*abort; ++n) {
        const int s = n % Lay::kVStages;
        const uint32_t u = n / Lay::kVStages;
        const int key0 = p.cached ? static_cast<int>(b * p.cache_stride) + sc.kt(n) * kBN : seq0 + sc.kt(n) * kBN;
        if (u > 0 && !mbar_wait(&bars->v_empty[s], (u - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], kTileTx);
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(sV + s * Lay::kTileBytes + bx * Lay::kBoxBytes, &tm_v, &bars->v_full[s], bx * 64, hkv, key0);
        issued[s] = static_cast<int>(u) + 1;
      }
      for (int s = 0; s < Lay::kVStages; ++s)
        if (issued[s] > 0) mbar_wait_bounded(&bars->v_full[s], (issued[s] - 1) & 1);
    }
  } else if (warp == 1) {
    give_regs();
    // ---------------------------------------------------------- MMA issuer
    const bool leader = elect_one();
    const uint64_t dq0 = sdesc_kmajor_sw128(smem_u32(sQ));
    const uint64_t dk0 = sdesc_kmajor_sw128(smem_u32(sK));
    const uint64_t dv0 = sdesc_mnmajor_sw128(smem_u32(sV), 16384);
    auto commit = [&](uint64_t* bar) {
      if (leader) umma_commit(bar);
    };
    // S(m) into buffer m & 1 (after PV(m - 2) read P(m - 2) there: issued earlier by this warp)
    auto s_visit = [&](int m) -> bool {
      if (sc.phase_start(m)) {
        if (!warp_wait(&bars->q_ready, m == 0 ? 0 : 1, abort)) return false;
        tc_fence_after();
      }
      const int ks = m % Lay::kKStages;
      if (!warp_wait(&bars->k_ready[ks], (m / Lay::kKStages) & 1, abort)) return false;
      tc_fence_after();
      const uint64_t kd = dk0 + static_cast<uint32_t>((ks * Lay::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const uint32_t off = (kk >> 2) * (Lay::kBoxBytes >> 4) + (kk & 3) * 2;
        if (leader) umma_ss(tmem + (m & 1) * 128, dq0 + off, kd + off, kIdescS, kk > 0);
      }
      commit(&bars->s_full[m & 1]);
      commit(&bars->k_empty[ks]);
      if (sc.phase_end(m)) commit(&bars->q_empty);
      return true;
    };
    bool ok = s_visit(0);
    if (ok && sc.n_virt > 1) ok = s_visit(1);
    for (int n = 0; n < sc.n_virt && ok; ++n) {
      JL_TRACE_AT(n, 0);
      if (!(ok = warp_wait(&bars->p_ready[n & 1], (n >> 1) & 1, abort))) break;
      JL_TRACE_AT(n, 1);
      tc_fence_after();
      const int vs = n % Lay::kVStages;
      if (!(ok = warp_wait(&bars->v_full[vs], (n / Lay::kVStages) & 1, abort))) break;
      JL_TRACE_AT(n, 2);
      const uint64_t vd = dv0 + static_cast<uint32_t>((vs * Lay::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < PSTEPS; ++kk)
        if (leader)
          umma_ts(tmem + Lay::kOCol, tmem + (n & 1) * 128 + kk * 8, vd + kk * (2048 >> 4), kIdescO,
                  (n > 0 || kk > 0) ? 1u : 0u);
      commit(&bars->v_empty[vs]);
      commit(&bars->pv_done);
      if (n + 2 < sc.n_virt) ok = s_visit(n + 2);
      JL_TRACE_AT(n, 3);
    }
    if (ok) commit(&bars->o_final);
    commit(&bars->teardown);
    mbar_wait_bounded(&bars->teardown, 0);
    __syncwarp();
  } else if (warp >= 8 && D == 128 && !p.cached) {
    setmaxnreg_dec<Lay::kRegsRot>();
    // --------------------------------- rotation, head_dim 128, keys from the prompt
    // 16-byte accesses (rotate_slice_v128): lane group q of warp rw starts at row
    // 16 rw + 4 q of the tile.
    const int rw = warp - 8;
    const int c8 = lane & 7, r4 = 16 * rw + 4 * (lane >> 3);
    auto anchor8 = [&](RotFactor8& f, int row, bool rt) {
      load_factor8(f, rt ? p.cos_rem : p.cos_tab, rt ? p.sin_rem : p.sin_tab, row,
                   (rt ? p.n_rem_rows : p.n_tab_rows) - 1, c8);
    };
    auto kgrp = [&](int n) { return (!interp && (sc.remote(n) || local_uses_remote)) ? G : 1; };
    const bool write_cache = p.k_cache_out != nullptr && slot == 0 && p.mode == 0;
    // Position of this lane's first key row in visit m, divided by that visit's g:
    // stepped from the previous visit (the next key tile is 128 positions on) and
    // divided afresh only when the tile sequence or g changes (phase starts).
    StepDiv kdiv;
    int kdiv_kt = -2, kdiv_g = 0;
    auto key_row = [&](int m, int& cnt) -> int {
      const int gm = kgrp(m), pos = sc.kt(m) * kBN + r4;
      if (gm == 1) {
        cnt = 0;
        return pos;
      }
      if (sc.kt(m) == kdiv_kt + 1 && gm == kdiv_g) kdiv.next();
      else kdiv.init(pos, kBN, gm);
      kdiv_kt = sc.kt(m);
      kdiv_g = gm;
      cnt = kdiv.r;
      return kdiv.q;
    };
    RotFactor8 st8, fk8_next;
    int cnt_next = 0;
    if (!p.krot) anchor8(fk8_next, key_row(0, cnt_next), interp && sc.remote(0));
    for (int n = 0; n < sc.n_virt; ++n) {
      const bool remote = sc.remote(n);
      const bool rem_tab = interp && remote;
      const int g = kgrp(n);
      if (sc.phase_start(n)) {
        anchor8(st8, 1, rem_tab);  // one row's step of the phase's table
        RotFactor8 fq8;
        const int qpos = sc.q_lo + r4;
        anchor8(fq8, g == 1 ? qpos : qpos / g, rem_tab);
        {
          const int first = sc.q_lo + RR * rw, last = min(first + RR - 1, L - 1);
          JL_CHECK(first > last || (last / g < (rem_tab ? p.n_rem_rows : p.n_tab_rows) &&
                                    (g == 1 || interp || last / g < p.w_pre)));
        }
        if (!mbar_wait(&bars->q_full, n == 0 ? 0 : 1, abort)) break;
        rotate_slice_v128_any(sQ, rw, sc.q_lo, g == 1 ? 0 : qpos % g, g, fq8, st8, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_ready);
      }
      const RotFactor8 fk8 = fk8_next;
      const int cnt_k = cnt_next;
      if (n + 1 < sc.n_virt && !p.krot) anchor8(fk8_next, key_row(n + 1, cnt_next), interp && sc.remote(n + 1));
      const int s = n % Lay::kKStages;
      {
        const int first = sc.kt(n) * kBN + RR * rw, last = min(first + RR - 1, L - 1);
        JL_CHECK(first > last || (last / g < (rem_tab ? p.n_rem_rows : p.n_tab_rows) &&
                                  (g == 1 || interp || last / g < p.w_pre)));
      }
      if (rw < 4) JL_TRACE_AT(n, 5 + 3 * rw);
      if (!mbar_wait(&bars->k_full[s], (n / Lay::kKStages) & 1, abort)) break;
      if (rw < 4) JL_TRACE_AT(n, 6 + 3 * rw);
      uint8_t* tile = sK + s * Lay::kTileBytes;
      if (!p.krot) rotate_slice_v128_any(tile, rw, sc.kt(n) * kBN, cnt_k, g, fk8, st8, lane);
      if (write_cache && !remote && sc.kt(n) == qt) {
        __syncwarp();
        write_cache_slice<D, RR>(tile, rw, p, b, qt * kBN, n_rows - qt * kBN, q_tok0, hkv, lane);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->k_ready[s]);
      if (rw < 4) JL_TRACE_AT(n, 7 + 3 * rw);
    }
  } else if (warp >= 8) {
    setmaxnreg_dec<Lay::kRegsRot>();
    // ------------------------------------------------------------ rotation
    const int rw = warp - 8;
    RotFactor<D> step, step_rem;
    load_factor<D>(step, p, 1, lane);
    if (interp) load_factor<D>(step_rem, p, 1, lane, true);
    StepDiv kdiv{};  // as in jl_prefill_kernel's rotation role
    int kdiv_kt = -2, kdiv_g = 0;
    auto key_anchor = [&](int m) -> int64_t {
      const int gm = p.cached ? G : ((sc.remote(m) || local_uses_remote) ? G : 1);
      const int pos = sc.kt(m) * kBN + RR * rw;
      if (gm == 1) return p.cached ? 0 : pos;
      if (sc.kt(m) == kdiv_kt + 1 && gm == kdiv_g) kdiv.next();
      else kdiv.init(pos, kBN, gm);
      kdiv_kt = sc.kt(m);
      kdiv_g = gm;
      return p.cached ? pos - kdiv.q : kdiv.q;
    };
    RotFactor<D> fk_next;
    if (!p.krot) load_factor<D>(fk_next, p, key_anchor(0), lane, interp && sc.remote(0));
    const bool write_cache = p.k_cache_out != nullptr && slot == 0 && p.mode == 0 && !p.cached;
    for (int n = 0; n < sc.n_virt; ++n) {
      const bool remote = sc.remote(n);
      const bool rem_tab = interp && remote;
      const int g = (!interp && (remote || local_uses_remote)) ? G : 1;
      const RotFactor<D>& stp = rem_tab ? step_rem : step;
      if (sc.phase_start(n)) {
        RotFactor<D> fq;
        load_factor<D>(fq, p, slice_anchor_row(sc.q_lo, rw, g, RR), lane, rem_tab);
        {
          const int first = sc.q_lo + RR * rw, last = min(first + RR - 1, L - 1);
          JL_CHECK(first > last || (last / g < (rem_tab ? p.n_rem_rows : p.n_tab_rows) &&
                                    (g == 1 || interp || last / g < p.w_pre)));
        }
        if (!mbar_wait(&bars->q_full, n == 0 ? 0 : 1, abort)) break;
        rotate_slice_any<D, RR>(sQ, rw, sc.q_lo, g, fq, stp, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_ready);
      }
      const RotFactor<D> fk = fk_next;
      if (n + 1 < sc.n_virt && !p.krot) load_factor<D>(fk_next, p, key_anchor(n + 1), lane, interp && sc.remote(n + 1));
      const int s = n % Lay::kKStages;
      {
        const int first = sc.kt(n) * kBN + RR * rw, last = min(first + RR - 1, L - 1);
        if (p.cached)
          JL_CHECK(first > last || g == 1 || last - last / G < p.n_tab_rows);
        else
          JL_CHECK(first > last || (last / g < (rem_tab ? p.n_rem_rows : p.n_tab_rows) &&
                                    (g == 1 || interp || last / g < p.w_pre)));
      }
      if (rw < 4) JL_TRACE_AT(n, 5 + 3 * rw);
      if (!mbar_wait(&bars->k_full[s], (n / Lay::kKStages) & 1, abort)) break;
      if (rw < 4) JL_TRACE_AT(n, 6 + 3 * rw);
      uint8_t* tile = sK + s * Lay::kTileBytes;
      if (p.krot) {
        // the keys arrived rotated for this visit's kind
      } else if (!p.cached) {
        rotate_slice_any<D, RR>(tile, rw, sc.kt(n) * kBN, g, fk, stp, lane);
        if (write_cache && !remote && sc.kt(n) == qt) {
          __syncwarp();
          write_cache_slice<D, RR>(tile, rw, p, b, qt * kBN, n_rows - qt * kBN, q_tok0, hkv, lane);
        }
      } else if (g > 1) {
        switch (g) {
          case 2: correct_slice<D, 2, RR>(tile, rw, sc.kt(n) * kBN, g, fk, step, lane); break;
          case 4: correct_slice<D, 4, RR>(tile, rw, sc.kt(n) * kBN, g, fk, step, lane); break;
          default: correct_slice<D, 0, RR>(tile, rw, sc.kt(n) * kBN, g, fk, step, lane); break;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->k_ready[s]);
      if (rw < 4) JL_TRACE_AT(n, 7 + 3 * rw);
    }
  } else if (warp >= 4) {
    setmaxnreg_inc<Lay::kRegsSoftmax>();
    // ------------------------------------------------------ softmax + epilogue
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int i = sc.q_lo + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t t_o = t_lane + Lay::kOCol;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < sc.n_virt; ++n) {
      const int buf = n & 1;
      const uint32_t t_s = t_lane + buf * 128;
      if (!(ok = mbar_wait(&bars->s_full[buf], (n >> 1) & 1, abort))) break;
      JL_TRACE_AT(n, 20 + 5 * wq);
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(t_s, sr);
      const bool msk = sc.masked(n);
      const int hi = i - sc.kt(n) * kBN;
      const int edge = hi - sc.w0;
      const bool rmt = sc.remote(n);
      const int keep_lo = msk ? (rmt ? -1 : edge) : -1;
      const int keep_hi = msk ? (rmt ? edge : hi) : kBN;
      float mx = -INFINITY;
      if (msk) {
#pragma unroll
        for (int e = 0; e < 128; ++e) mx = (e > keep_lo && e <= keep_hi) ? fmaxf(mx, __uint_as_float(sr[e])) : mx;
      } else {
        float m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; e += 8) {
          mx = fmax3(mx, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
          m1 = fmax3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
          m2 = fmax3(m2, __uint_as_float(sr[e + 4]), __uint_as_float(sr[e + 5]));
          m3 = fmax3(m3, __uint_as_float(sr[e + 6]), __uint_as_float(sr[e + 7]));
        }
        mx = fmaxf(fmaxf(mx, m1), fmaxf(m2, m3));
      }
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool resc = (m_run != -INFINITY) && (m_new > m_run + 8.f);
      const float alpha = resc ? ex2_approx(m_run - m_new) : 1.f;
      if (resc || m_run == -INFINITY) m_run = m_new;
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      JL_TRACE_AT(n, 21 + 5 * wq);
      float lsum = 0.f, lsum2 = 0.f;
      uint32_t pk[64];
      if (msk) softmax_chunk<true, 128, JL_DB_POLY>(sr, pk, 0, sl2, -m_use, keep_lo, keep_hi, lsum, lsum2);
      else softmax_chunk<false, 128, JL_DB_POLY>(sr, pk, 0, sl2, -m_use, keep_lo, keep_hi, lsum, lsum2);
      JL_TRACE_AT(n, 22 + 5 * wq);
      tmem_st64(t_s, pk);
      lsum += lsum2;
      l_run = l_run * alpha + lsum;
      // O *= alpha for the rows whose max moved: PV(n - 1) has to be complete (it is
      // issued when P(n - 1) is ready and may still be running), and PV(n) waits for
      // this tile's p_ready, so the rescale falls between them.
      if (__any_sync(0xffffffffu, resc)) {
        if (!(ok = mbar_wait(&bars->pv_done, (n - 1) & 1, abort))) break;
        tc_fence_after();
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
      mbar_arrive(&bars->p_ready[buf]);
      JL_TRACE_AT(n, 23 + 5 * wq);
    }
    if (ok && mbar_wait(&bars->o_final, 0, abort)) {
      tc_fence_after();
      const bool valid = i <= sc.q_hi;
      JL_CHECK(!valid || (static_cast<int64_t>(q_tok0) + row < p.total_tokens && h < p.Hq));
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const int64_t row_off = ((static_cast<int64_t>(q_tok0) + row) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        if (valid && p.out_f32 != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.out_f32 + row_off + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(o[4 * v4]) * inv, __uint_as_float(o[4 * v4 + 1]) * inv,
                                  __uint_as_float(o[4 * v4 + 2]) * inv, __uint_as_float(o[4 * v4 + 3]) * inv);
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + row_off + c * 32);
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
        const float m_fin = (m_run == -INFINITY) ? 0.f : m_run;
        p.lse[static_cast<int64_t>(h) * p.total_tokens + q_tok0 + row] = (m_fin + log2f(l_run)) * 0.69314718055994531f;
      }
    }
  }

  if (warp == 3) give_regs();  // the control warpgroup's idle warp still gives its share

  // ---- teardown: every role is done; TMEM is released by its allocator warp ----
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

// Literal inclusion-exclusion merge of the three passes (natural-log LSEs):
//   M = max(lse1, lse2); a_p = e^(lse_p - M) (0 for an empty pass);
//   Z = a1 + a2 - a3;  out = (a1 O1 + a2 O2 - a3 O3) / Z;  lse = M + ln Z.
// One warp per (token, head) row.
template <int D>
__global__ void __launch_bounds__(256) jl_ie_merge_kernel(const float* __restrict__ o3x,
                                                          const float* __restrict__ lse3x, int64_t T, int Hq,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (row >= T * Hq) return;
  const int64_t t = row / Hq;
  const int h = static_cast<int>(row % Hq);
  const int64_t plane = T * Hq * D;
  const float l1 = lse3x[static_cast<int64_t>(h) * T + t];
  const float l2 = lse3x[T * Hq + static_cast<int64_t>(h) * T + t];
  const float l3 = lse3x[2 * T * Hq + static_cast<int64_t>(h) * T + t];
  const float M = fmaxf(l1, l2);
  const float a1 = l1 == -INFINITY ? 0.f : __expf(l1 - M);
  const float a2 = l2 == -INFINITY ? 0.f : __expf(l2 - M);
  const float a3 = l3 == -INFINITY ? 0.f : __expf(l3 - M);
  const float Z = a1 + a2 - a3;
  const float inv = 1.f / Z;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) {
    const int64_t c = row * D + lane * (D / 32) + e;
    const float v = a1 * o3x[c] + a2 * o3x[plane + c] - a3 * o3x[2 * plane + c];
    out[c] = __float2bfloat16_rn(v * inv);
  }
  if (lane == 0 && lse != nullptr) lse[static_cast<int64_t>(h) * T + t] = M + __logf(Z);
}

}  // namespace jl
