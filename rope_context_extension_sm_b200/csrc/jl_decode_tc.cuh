// jl_decode_tc.cuh -- split-K bifocal decode on sm_100a with the keys on the
// tensor-core M dimension (head_dim 128, up to 16 query heads per KV head; the
// template GROUP is a capacity of 1, 2, 4, 8 or 16 heads and the runtime group
// p.group <= GROUP picks the rows that hold real queries).
//
// Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
// RoPE", Methodology section 2, on-the-fly correction rotation.  The cache holds
// base keys k~_j = R(j) k_j and is only read.  Remote keys (i - j >= w0) score
// <R(f(i) - i) q~, R(f(j) - j) k~_j> = <R(f(i)) q, R(f(j)) k_j>; local keys score
// <q~, k~_j>.
//
// CTA = (KV head, chunk of keys, batch entry).  The caches are contiguous per
// entry, or a page pool with a block table (pages of a multiple of 128 keys, so a
// tile lies in one page).  Per 128-key tile:
//   warp 0      TMA producer: raw K and V tiles (3 stages)
//   warp 1      TMEM allocator + tcgen05.mma issuer (warp-uniform loop, one
//               elected lane issues, descriptors formed once)
//   warps 2-3,  correction warps (16, or 8 for 16 heads per KV head): rotate
//   8..         the remote rows of the K tile in place by R(-(j - f(j)))
//               (cos/sin stepped along the rows by complex
//               multiplication, anchored on a table row prefetched a tile ahead)
//   warps 4-7   softmax, thread = key row of S^T and channel row of O^T
// MMAs:  S^T[128 keys x 32] = K_tile . [R(f(i)-i) q~ (16 rows) | q~ (16 rows)]^T
//        O^T[128 ch x 16]  += V_tile^T . P^T          (A = V tile, MN-major)
// Each key row picks the remote or the local half of its S^T row, so the tile
// that straddles the window edge needs no second visit.  Per-head maxima are
// reduced across the 128 threads each tile; row sums stay per thread and are
// reduced once at the end.  The partial (m, l, o) per query head goes to the
// workspace.  With p.counters set, the last CTA of each (entry, KV head) to finish
// merges that head group's partials itself (one launch per decode); otherwise
// jl_decode_combine_kernel merges them.
#pragma once

#include "jl_decode.cuh"
#include "jl_device.cuh"

namespace jl {

// Optional timeline of one CTA (built only with -DJL_TRACE, for measurements):
// SM clock stamps of the roles' events on the first 64 tiles of CTA (0, 1, 0).
#ifdef JL_TRACE
__device__ long long g_trace_dec[64 * 16];
#define JL_DTRACE_AT(n, slot)                                                                           \
  do {                                                                                                  \
    if (blockIdx.x == 0 && blockIdx.y == 1 && blockIdx.z == 0 && (n) < 64 && (threadIdx.x & 31) == 0) \
      g_trace_dec[(n) * 16 + (slot)] = clock64();                                                       \
  } while (0)
#else
#define JL_DTRACE_AT(n, slot) \
  do {                        \
  } while (0)
#endif

constexpr int kDecTile = 128;    // keys per tile
constexpr int kDecStages = 3;    // K/V pipeline depth
constexpr int kDecQRows = 32;    // B operand rows of the score MMA (16 remote + 16 local)
constexpr int kDecHeads = 16;    // N of the PV MMA (query heads per KV head, padded)

template <int GROUP>
struct DecTcLayout {
  static constexpr int kTile = kDecTile * 128 * 2;          // 32 KB (K or V tile)
  static constexpr int kK = 0;
  static constexpr int kV = kK + kDecStages * kTile;
  static constexpr int kQ = kV + kDecStages * kTile;        // [32][128] bf16 = 8 KB (2 boxes of 4 KB)
  static constexpr int kP = kQ + kDecQRows * 256;           // 2 x [16][128] bf16 = 2 x 4 KB
  static constexpr int kRed = kP + 2 * kDecHeads * 256;     // reductions: float [4][16] x 2
  static constexpr int kBar = kRed + 1024;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 128;  // S^T x2 (64) + O^T (16)
  // correction warps: 16 (8 rows each) unless 16 query heads per KV head make the
  // softmax warps register-heavy, then 8 (16 rows each)
  static constexpr int kRotWarps = GROUP <= 8 ? 16 : 8;
  static constexpr int kRotRows = kDecTile / kRotWarps;
  static constexpr int kThreads = 32 * (6 + kRotWarps);
};

struct DecTcBars {
  uint64_t k_full[kDecStages], k_ready[kDecStages], k_empty[kDecStages];
  uint64_t v_full[kDecStages], v_empty[kDecStages];
  uint64_t s_full[2], p_ready[2], pv_done, q_ready, teardown;
  uint64_t red_full[2], red_end;  // softmax-warp exchanges (bounded, unlike bar.sync)
  uint64_t fin;                   // the partials of every softmax thread are written
  uint32_t tmem_base;
  int abort;
  int last;                       // this CTA merges its head group's partials
};

// Ticket of one split CTA of an (entry, KV head): true for the last of its n CTAs.
// Two 8-byte words per (entry, KV head), neither of which has to start cleared:
//  - words[0] holds (kTicketClean << 32) | count once in use.  Each CTA adds 1 (one
//    atomic, no retries); the one that finds count n - 1 is last and puts the word
//    back to (kTicketClean, 0) -- every add of the call is in by then -- so the next
//    call, or a graph replaying this one, finds it clear.
//  - A words[0] without the marker (a workspace never used by a decode) sends every
//    CTA of the call (all of them add to the same unmarked word) to words[1].  That
//    word holds (tag << 32) | count, tag = the call's p.epoch, and a word with another
//    tag counts as zero; it is advanced by compare-and-swap, bounded since each failed
//    exchange means another CTA's succeeded.  Its last CTA marks words[0].
// The atomics are acquire-release at GPU scope: they publish every store the calling
// thread has observed (the CTA's partials, ordered before it by an mbarrier) and, for
// the last CTA, make the other CTAs' partials visible.
constexpr uint32_t kTicketClean = 0x4a4c3136u;
constexpr unsigned long long kTicketCleanWord = static_cast<unsigned long long>(kTicketClean) << 32;

__device__ __forceinline__ unsigned long long add_acq_rel(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

__device__ __forceinline__ unsigned long long cas_acq_rel(unsigned long long* p, unsigned long long cmp,
                                                          unsigned long long val) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.cas.b64 %0, [%1], %2, %3;" : "=l"(old) : "l"(p), "l"(cmp), "l"(val)
               : "memory");
  return old;
}

__device__ __forceinline__ void store_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ bool take_ticket(unsigned long long* words, uint32_t tag, int n) {
  const unsigned long long old = add_acq_rel(words, 1ull);
  if (static_cast<uint32_t>(old >> 32) == kTicketClean) {
    const bool last = static_cast<uint32_t>(old) + 1u >= static_cast<uint32_t>(n);
    if (last) store_relaxed(words, kTicketCleanWord);
    return last;
  }
  unsigned long long cur;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(cur) : "l"(words + 1) : "memory");
  for (int tries = 0; tries < 4 * n + 64; ++tries) {
    const uint32_t cnt = (static_cast<uint32_t>(cur >> 32) == tag) ? static_cast<uint32_t>(cur) + 1u : 1u;
    const bool last = cnt >= static_cast<uint32_t>(n);
    const unsigned long long want = (static_cast<unsigned long long>(tag) << 32) | (last ? 0u : cnt);
    const unsigned long long seen = cas_acq_rel(words + 1, cur, want);
    if (seen == cur) {
      if (last) store_relaxed(words, kTicketCleanWord);
      return last;
    }
    cur = seen;
  }
  atomicOr(&g_status, kDevErrTimeout);
  return false;
}

// Merge of the ns split partials of query heads [hk * ng, hk * ng + ng) of entry b,
// by all nthreads threads of the last CTA.  The same log-sum-exp blend as
// jl_decode_combine_kernel.  Item = (head, channel pair); lanes l and l ^ 16 of a warp
// take the first and the second half of the splits, each with a running maximum, and
// join through a shuffle, so up to 2 * kMergeBatch splits take one round of loads.
// Partials written by other CTAs in this launch are read through L2 (ld.global.cg).
constexpr int kMergeBatch = 8;
__device__ __forceinline__ void merge_head_group(const DecodeParams& p, int b, int hk, int ng, int ns,
                                                 int nthreads, bool failed) {
  // A CTA that gave up set the status word before its ticket, so this read (after the
  // last ticket's acquire) sees it; it is issued with the partials and used last.
  const unsigned status = *reinterpret_cast<volatile unsigned*>(&g_status);
  const int64_t sstride = static_cast<int64_t>(p.Hq) * (128 + 2);
  const int half_ns = (ns + 1) / 2, n_items = ng * 64;
  const int lane = threadIdx.x & 31, half = lane >> 4;
  for (int first = (threadIdx.x >> 5) * 16; first < n_items; first += (nthreads >> 5) * 16) {  // per warp
    const int it = min(first + (lane & 15), n_items - 1);
    const int h = hk * ng + (it >> 6), cp = (it & 63) * 2;
    const float* base = p.ws + (static_cast<int64_t>(b) * p.n_split * p.Hq + h) * (128 + 2);
    const int s_lo = half * half_ns, s_hi = min(ns, s_lo + half_ns);
    float M = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f;
    for (int s0 = s_lo; s0 < s_hi; s0 += kMergeBatch) {
      float ms[kMergeBatch], ls[kMergeBatch];
      float2 os[kMergeBatch];
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u) {  // past s_hi: the last split again, skipped below
        const float* ps = base + min(s0 + u, s_hi - 1) * sstride;
        ms[u] = __ldcg(ps);
        ls[u] = __ldcg(ps + 1);
        os[u] = __ldcg(reinterpret_cast<const float2*>(ps + 2 + cp));
      }
      float mb = M;
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u)
        if (s0 + u < s_hi) mb = fmaxf(mb, ms[u]);
      if (mb == -INFINITY) continue;
      if (mb > M) {  // rescale what is summed so far to the new maximum
        const float r = (M == -INFINITY) ? 0.f : ex2_approx(M - mb);
        l *= r;
        a0 *= r;
        a1 *= r;
        M = mb;
      }
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u) {
        const float sc = (s0 + u < s_hi && ms[u] != -INFINITY) ? ex2_approx(ms[u] - M) : 0.f;
        l = fmaf(ls[u], sc, l);
        a0 = fmaf(os[u].x, sc, a0);
        a1 = fmaf(os[u].y, sc, a1);
      }
    }
    // join the two halves (lane l ^ 16 holds the other one)
    const float Mo = __shfl_xor_sync(0xffffffffu, M, 16), lo_ = __shfl_xor_sync(0xffffffffu, l, 16);
    const float a0o = __shfl_xor_sync(0xffffffffu, a0, 16), a1o = __shfl_xor_sync(0xffffffffu, a1, 16);
    const float Mx = fmaxf(M, Mo);
    const float r = (M == -INFINITY) ? 0.f : ex2_approx(M - Mx), ro = (Mo == -INFINITY) ? 0.f : ex2_approx(Mo - Mx);
    l = l * r + lo_ * ro;
    a0 = a0 * r + a0o * ro;
    a1 = a1 * r + a1o * ro;
    if (half == 0 && first + lane < n_items) {
      // a split gave up: its partials are stale, so the output is marked undefined
      const bool bad = failed || (status & kDevErrTimeout) != 0;
      const float nan = __int_as_float(0x7fc00000);
      *reinterpret_cast<uint32_t*>(p.out + (static_cast<int64_t>(b) * p.Hq + h) * 128 + cp) =
          bad ? pack_bf16x2(nan, nan) : pack_bf16x2(a0 / l, a1 / l);
      if (cp == 0 && p.lse != nullptr)
        p.lse[static_cast<int64_t>(b) * p.Hq + h] = bad ? nan : (Mx + log2f(l)) * 0.69314718055994531f;
    }
  }
}

// warps 2-3 and 8.. correct keys; 4-7 (one TMEM lane quarter each) run the softmax
__device__ __forceinline__ int dec_rot_index(int warp) {
  return warp == 2 ? 0 : warp == 3 ? 1 : (warp >= 8 ? warp - 6 : -1);
}

// Rotate row r of a swizzled [128][128] bf16 tile in place by R(-n), f = (cos n theta, sin n theta).
__device__ __forceinline__ void rotate_row_neg(uint8_t* tile, int r, const float (&c)[2], const float (&s)[2],
                                               int lane) {
  const int off = r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + ((lane & 3) << 2);
  uint32_t* plo = reinterpret_cast<uint32_t*>(tile + off);
  uint32_t* phi = reinterpret_cast<uint32_t*>(tile + 16384 + off);
  const float2 a = unpack_bf16x2(*plo);
  const float2 b = unpack_bf16x2(*phi);
  // ya = a c + b s, yb = b c - a s on packed pairs (two frequencies per instruction)
  const uint64_t c2 = f2_pack(c[0], c[1]), s2 = f2_pack(s[0], s[1]);
  const uint64_t a2 = f2_pack(a.x, a.y), b2 = f2_pack(b.x, b.y);
  float2 ya, yb;
  f2_unpack(f2_fma(b2, s2, f2_mul(a2, c2)), ya.x, ya.y);
  f2_unpack(f2_sub(f2_mul(b2, c2), f2_mul(a2, s2)), yb.x, yb.y);
  *plo = pack_bf16x2(ya.x, ya.y);
  *phi = pack_bf16x2(yb.x, yb.y);
}

// (c, s) <- (c, s) * e^{i theta} when adv, else unchanged (select, no branch).
__device__ __forceinline__ void step_factor(float (&c)[2], float (&s)[2], const float (&st_c)[2],
                                            const float (&st_s)[2], bool adv) {
  const uint64_t c2 = f2_pack(c[0], c[1]), s2 = f2_pack(s[0], s[1]);
  const uint64_t tc2 = f2_pack(st_c[0], st_c[1]), ts2 = f2_pack(st_s[0], st_s[1]);
  float nc[2], ns[2];
  f2_unpack(f2_sub(f2_mul(c2, tc2), f2_mul(s2, ts2)), nc[0], nc[1]);
  f2_unpack(f2_fma(c2, ts2, f2_mul(s2, tc2)), ns[0], ns[1]);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    c[e] = adv ? nc[e] : c[e];
    s[e] = adv ? ns[e] : s[e];
  }
}

// Correct the remote rows (r <= last_remote) of an ROWS-row slice of keys j0 ..:
// R(-n_j), n_j = j - floor(j / G).  n steps by one per row except where f steps up
// (row r with (j0 + r + 1) % G == 0).  GS = G in {2, 4, 8} with j0 % G == 0 makes
// those rows compile-time; GS = 0 starts from j0_mod_g = j0 mod G (unused otherwise).
template <int ROWS, int GS>
__device__ __forceinline__ void correct_slice(uint8_t* slice, int j0_mod_g, int G, int last_remote, bool full,
                                              float (&fc)[2], float (&fs)[2], const float (&st_c)[2],
                                              const float (&st_s)[2], int lane) {
  if constexpr (GS > 0) {
    if (full) {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        rotate_row_neg(slice, r, fc, fs, lane);
        if ((r + 1) % GS != 0) step_factor(fc, fs, st_c, st_s, true);
      }
    } else {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        if (r <= last_remote) rotate_row_neg(slice, r, fc, fs, lane);
        if ((r + 1) % GS != 0) step_factor(fc, fs, st_c, st_s, true);
      }
    }
  } else {
    // Any G: bit r of adv says whether n steps after row r (it does unless
    // (j0 + r + 1) % G == 0), computed once per slice so the row loop carries no
    // counter; the partial-slice test is hoisted out of the loop like above.
    uint32_t adv = 0;
    int cnt = j0_mod_g;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      cnt = (cnt + 1 == G) ? 0 : cnt + 1;
      adv |= (cnt != 0 ? 1u : 0u) << r;
    }
    if (full) {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        rotate_row_neg(slice, r, fc, fs, lane);
        step_factor(fc, fs, st_c, st_s, (adv >> r) & 1u);
      }
    } else {
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        if (r <= last_remote) rotate_row_neg(slice, r, fc, fs, lane);
        step_factor(fc, fs, st_c, st_s, (adv >> r) & 1u);
      }
    }
  }
}

// Element (row, ch) of a 128-byte-swizzled K-major [rows][128] bf16 operand whose
// 64-channel boxes are box_bytes apart.
__device__ __forceinline__ int swz_off(int row, int ch, int box_bytes) {
  const int cc = ch & 63;
  return (ch >> 6) * box_bytes + row * 128 + ((((cc * 2) >> 4) ^ (row & 7)) << 4) + ((cc * 2) & 15);
}

template <int GROUP, bool PLAIN>
__global__ void __launch_bounds__(DecTcLayout<GROUP>::kThreads, 1)
    jl_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeParams p) {
  using Lay = DecTcLayout<GROUP>;
  constexpr uint32_t kTileTx = kDecTile * 128 * 2;
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, kDecQRows, false, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, kDecHeads, true, false);
  static_assert(GROUP <= kDecHeads, "up to 16 query heads per KV head");

  const int hk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int ng = p.group;  // query heads of this KV head (<= GROUP; the rest of the capacity is zero rows)
  // The next kernel in the stream may be scheduled now: it sets itself up and waits for
  // this whole grid before it reads anything (the combine step, or the next decode).
  griddep_launch_dependents();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sK = smem + Lay::kK;
  uint8_t* sV = smem + Lay::kV;
  uint8_t* sQ = smem + Lay::kQ;
  uint8_t* sP = smem + Lay::kP;
  float* red = reinterpret_cast<float*>(smem + Lay::kRed);  // [2][4][16]
  DecTcBars* bars = reinterpret_cast<DecTcBars*>(smem + Lay::kBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Setup that touches only this CTA's shared and tensor memory runs before the wait
  // for the previous kernel, so it overlaps that kernel's tail.
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_ready[s], Lay::kRotWarps);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_ready[t], 128);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->q_ready, 128);
    mbar_init(&bars->teardown, 1);
    mbar_init(&bars->red_full[0], 128);
    mbar_init(&bars->red_full[1], 128);
    mbar_init(&bars->red_end, 128);
    mbar_init(&bars->fin, 128);
    bars->abort = 0;
    bars->last = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Lay::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  griddep_wait();  // the query, the cache rows and the lengths may come from the previous kernel
  // One thread decides whether this CTA works (its keys exist, and no kernel has given up
  // on a bounded wait), so that the whole CTA takes the same path.
  if (threadIdx.x == 0) bars->last = (split * p.chunk >= p.seqlens[b]) ? 2 : status_failed() ? 1 : 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int L = p.seqlens[b];
  const int c0 = split * p.chunk;
  const int n_active = (L + p.chunk - 1) / p.chunk;  // split CTAs of (b, hk) that write partials
  if (bars->last != 0) {
    // Past the entry's length: nothing to do.  After a failure: skip the work, but still
    // take the ticket so that the last CTA marks the output undefined and the counter
    // is left clear.
    const bool failed = bars->last == 1;
    __syncthreads();
    if (failed && p.counters != nullptr) {
      if (threadIdx.x == 0) bars->last = take_ticket(p.counters + 2 * (b * p.Hkv + hk), p.epoch, n_active);
      __syncthreads();
      if (bars->last) merge_head_group(p, b, hk, ng, n_active, Lay::kThreads, true);
    }
    if (warp == 1) tmem_dealloc(tmem, Lay::kTmemCols);
    return;
  }
  const int c1 = min(c0 + p.chunk, L);
  const int n_tiles = (c1 - c0 + kDecTile - 1) / kDecTile;
  const int i = L - 1;
  int G = 1, jb = -1;  // remote keys are j <= jb
  if (!PLAIN) {
    G = max(1, (L + p.w_pre - 1) / p.w_pre);
    if (G > 1) jb = i - p.w0;
  }
  const int64_t row0 = static_cast<int64_t>(b) * p.cache_stride;  // token row of this entry's first key
  // the grid covers the length; the query's correction row is in the table
  JL_CHECK(L <= p.n_split * p.chunk && i < p.n_tab_rows && (i - i / G) < p.n_tab_rows && hk * ng + ng <= p.Hq);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued[kDecStages] = {0};
      StepDiv pdiv{};  // page and row of the tile's first key, stepped per tile (paged caches)
      if (p.block_table != nullptr) pdiv.init(c0, kDecTile, p.page_size);
      for (int n = 0; n < n_tiles && !*abort; ++n) {
        const int s = n % kDecStages;
        const uint32_t u = n / kDecStages;
        const int kpos = c0 + n * kDecTile;  // key position in entry b; a tile never crosses a page
        const int key0 = p.block_table != nullptr
                             ? p.block_table[static_cast<int64_t>(b) * p.max_pages + pdiv.q] * p.page_size + pdiv.r
                             : static_cast<int>(row0) + kpos;
        // contiguous: the tile's keys lie in entry b; paged: its page is inside the pool
        JL_CHECK(kpos < L && (p.block_table != nullptr
                                  ? (pdiv.q < p.max_pages && key0 >= 0 && key0 + kDecTile <= p.cache_stride)
                                  : L <= p.cache_stride));
        if (p.block_table != nullptr) pdiv.next();
        JL_DTRACE_AT(n, 0);
        if (u > 0 && !mbar_wait(&bars->k_empty[s], (u - 1) & 1, abort)) break;
        JL_DTRACE_AT(n, 1);
        mbar_arrive_expect_tx(&bars->k_full[s], kTileTx);
        tma_load_3d(sK + s * Lay::kTile, &tm_k, &bars->k_full[s], 0, hk, key0);
        tma_load_3d(sK + s * Lay::kTile + 16384, &tm_k, &bars->k_full[s], 64, hk, key0);
        if (u > 0 && !mbar_wait(&bars->v_empty[s], (u - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], kTileTx);
        tma_load_3d(sV + s * Lay::kTile, &tm_v, &bars->v_full[s], 0, hk, key0);
        tma_load_3d(sV + s * Lay::kTile + 16384, &tm_v, &bars->v_full[s], 64, hk, key0);
        issued[s] = static_cast<int>(u) + 1;
      }
      for (int s = 0; s < kDecStages; ++s)
        if (issued[s] > 0) {
          mbar_wait_bounded(&bars->k_full[s], (issued[s] - 1) & 1);
          mbar_wait_bounded(&bars->v_full[s], (issued[s] - 1) & 1);
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs the loop, so every operand stays warp-uniform, and one
    // elected lane issues each tcgen05 instruction.  Descriptors are formed once:
    // the descriptor of (base + off) is that of base plus off / 16 (the start-address
    // field, which cannot carry below 256 KB of shared memory).
    const bool leader = elect_one();
    const uint64_t dk0 = sdesc_kmajor_sw128(smem_u32(sK));
    const uint64_t dv0 = sdesc_mnmajor_sw128(smem_u32(sV), 16384);
    const uint64_t dq0 = sdesc_kmajor_sw128(smem_u32(sQ));
    const uint64_t dp0 = sdesc_kmajor_sw128(smem_u32(sP));
    auto issue_s = [&](int n) {
      const uint64_t kd = dk0 + static_cast<uint32_t>(((n % kDecStages) * Lay::kTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off_k = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        const uint32_t off_q = ((kk >> 2) * (kDecQRows * 128) + (kk & 3) * 32) >> 4;
        if (leader) umma_ss(tmem + (n & 1) * 32, kd + off_k, dq0 + off_q, kIdescS, kk > 0);
      }
    };
    auto issue_pv = [&](int n) {
      const uint64_t vd = dv0 + static_cast<uint32_t>(((n % kDecStages) * Lay::kTile) >> 4);
      const uint64_t pd = dp0 + static_cast<uint32_t>(((n & 1) * (kDecHeads * 256)) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off_p = ((kk >> 2) * (kDecHeads * 128) + (kk & 3) * 32) >> 4;
        if (leader) umma_ss(tmem + 64, vd + ((kk * 2048) >> 4), pd + off_p, kIdescO, (n > 0 || kk > 0) ? 1u : 0u);
      }
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) umma_commit(bar);
    };
    bool ok = warp_wait(&bars->q_ready, 0, abort);
    if (ok) {
      tc_fence_after();
      ok = warp_wait(&bars->k_ready[0], 0, abort);
    }
    if (ok) {
      tc_fence_after();
      issue_s(0);
      commit(&bars->s_full[0]);
      commit(&bars->k_empty[0]);
    }
    for (int n = 0; n < n_tiles && ok; ++n) {
      if (n + 1 < n_tiles) {  // scores of the next tile overlap this tile's softmax
        const int s1 = (n + 1) % kDecStages;
        if (!(ok = warp_wait(&bars->k_ready[s1], ((n + 1) / kDecStages) & 1, abort))) break;
        tc_fence_after();
        issue_s(n + 1);
        JL_DTRACE_AT(n + 1, 5);
        commit(&bars->s_full[(n + 1) & 1]);
        commit(&bars->k_empty[s1]);
      }
      if (!(ok = warp_wait(&bars->p_ready[n & 1], (n >> 1) & 1, abort))) break;
      tc_fence_after();
      const int s = n % kDecStages;
      if (!(ok = warp_wait(&bars->v_full[s], (n / kDecStages) & 1, abort))) break;
      JL_DTRACE_AT(n, 4);
      issue_pv(n);
      commit(&bars->pv_done);
      commit(&bars->v_empty[s]);
    }
    // Every issued MMA must finish before TMEM is released.
    commit(&bars->teardown);
    mbar_wait_bounded(&bars->teardown, 0);
    __syncwarp();
  } else if (dec_rot_index(warp) >= 0) {
    // ---------------------------------------------------- correction warps
    const int rw = dec_rot_index(warp);
    float st_c[2], st_s[2];  // e^{i theta_c}
    {
      const float2 cc = __ldg(reinterpret_cast<const float2*>(p.cos_tab + 64 + 2 * lane));
      const float2 ss = __ldg(reinterpret_cast<const float2*>(p.sin_tab + 64 + 2 * lane));
      st_c[0] = cc.x; st_c[1] = cc.y; st_s[0] = ss.x; st_s[1] = ss.y;
    }
    // j / G for this warp's first key, stepped from tile to tile (one division here;
    // a division per tile would queue on the MUFU unit behind the softmax).
    StepDiv jdiv{};
    if (G > 1) jdiv.init(c0 + Lay::kRotRows * rw, kDecTile, G);
    // anchor of tile n (called for n = 0, 1, 2, ... in order); rem = j mod G of its first key
    auto anchor = [&](int n, float (&c)[2], float (&s)[2], int& rem) {
      const int j = c0 + n * kDecTile + Lay::kRotRows * rw;
      int64_t row = G > 1 ? j - jdiv.q : 0;  // correction index n_j = j - f(j)
      rem = G > 1 ? jdiv.r : 0;
      if (G > 1) jdiv.next();
      {
        const int last = min(j + Lay::kRotRows - 1, c1 - 1);  // rows of the valid keys of this slice
        JL_CHECK(j > last || last - last / G < p.n_tab_rows);
      }
      row = row > p.n_tab_rows - 1 ? p.n_tab_rows - 1 : row;
      const float2 cc = ldg_now_f2(p.cos_tab + row * 64 + 2 * lane);  // a tile ahead: issued here
      const float2 ss = ldg_now_f2(p.sin_tab + row * 64 + 2 * lane);
      c[0] = cc.x; c[1] = cc.y; s[0] = ss.x; s[1] = ss.y;
    };
    float nc[2], ns[2];
    int nrem = 0;
    anchor(0, nc, ns, nrem);
    for (int n = 0; n < n_tiles; ++n) {
      float fc[2] = {nc[0], nc[1]}, fs[2] = {ns[0], ns[1]};
      const int rem = nrem;
      if (n + 1 < n_tiles) anchor(n + 1, nc, ns, nrem);
      const int s = n % kDecStages;
      if (!mbar_wait(&bars->k_full[s], (n / kDecStages) & 1, abort)) break;
      if (rw == 0) JL_DTRACE_AT(n, 2);
      const int j0 = c0 + n * kDecTile + Lay::kRotRows * rw;  // key of this warp's first row
      const int last_remote = min(jb, c1 - 1) - j0;             // rows r <= last_remote are remote
      if (last_remote >= 0) {
        uint8_t* slice = sK + s * Lay::kTile + Lay::kRotRows * rw * 128;
        const bool full = last_remote >= Lay::kRotRows - 1;  // else the slice straddles the window edge
        switch (G) {  // slices start at multiples of 8 keys: for G | 8 the step rows are fixed
          case 2: correct_slice<Lay::kRotRows, 2>(slice, j0, G, last_remote, full, fc, fs, st_c, st_s, lane); break;
          case 4: correct_slice<Lay::kRotRows, 4>(slice, j0, G, last_remote, full, fc, fs, st_c, st_s, lane); break;
          case 8: correct_slice<Lay::kRotRows, 8>(slice, j0, G, last_remote, full, fc, fs, st_c, st_s, lane); break;
          default: correct_slice<Lay::kRotRows, 0>(slice, rem, G, last_remote, full, fc, fs, st_c, st_s, lane); break;
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->k_ready[s]);
      if (rw == 0) JL_DTRACE_AT(n, 3);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int wq = warp - 4;  // 0..3: TMEM lane quarter
    const int tid = threadIdx.x - 128;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    // Query operand: rows 0..15 remote-corrected R(f(i) - i) q~, rows 16..31 q~; zero padding.
    // Thread = (head g, channels c..c+7 and c+64..c+71): all of its loads (two 16-byte
    // query words, and for G > 1 the correction row's cos/sin) go out before any is used.
    {
      const int g = tid >> 3, c = (tid & 7) * 8;
      uint4 qlo = make_uint4(0, 0, 0, 0), qhi = qlo;
      float4 c0v = make_float4(0.f, 0.f, 0.f, 0.f), c1v = c0v, s0v = c0v, s1v = c0v;
      if (g < ng) {
        const __nv_bfloat16* qp = p.q + (static_cast<int64_t>(b) * p.Hq + hk * ng + g) * 128 + c;
        qlo = *reinterpret_cast<const uint4*>(qp);
        qhi = *reinterpret_cast<const uint4*>(qp + 64);
        if (G > 1 && !PLAIN) {
          const int64_t nq = i - i / G;  // correction index of the query
          const float4* cp = reinterpret_cast<const float4*>(p.cos_tab + nq * 64 + c);
          const float4* sp = reinterpret_cast<const float4*>(p.sin_tab + nq * 64 + c);
          c0v = cp[0];
          c1v = cp[1];
          s0v = sp[0];
          s1v = sp[1];
        }
      }
      const uint32_t lw[4] = {qlo.x, qlo.y, qlo.z, qlo.w}, hw[4] = {qhi.x, qhi.y, qhi.z, qhi.w};
      uint32_t rlo[4] = {lw[0], lw[1], lw[2], lw[3]}, rhi[4] = {hw[0], hw[1], hw[2], hw[3]};
      if (G > 1 && !PLAIN) {
        const float cs[8] = {c0v.x, c0v.y, c0v.z, c0v.w, c1v.x, c1v.y, c1v.z, c1v.w};
        const float sn[8] = {s0v.x, s0v.y, s0v.z, s0v.w, s1v.x, s1v.y, s1v.z, s1v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // (lo, hi) -> (lo c + hi s, hi c - lo s), channels 2e, 2e + 1
          const float2 a = unpack_bf16x2(lw[e]), bb = unpack_bf16x2(hw[e]);
          rlo[e] = pack_bf16x2(a.x * cs[2 * e] + bb.x * sn[2 * e], a.y * cs[2 * e + 1] + bb.y * sn[2 * e + 1]);
          rhi[e] = pack_bf16x2(bb.x * cs[2 * e] - a.x * sn[2 * e], bb.y * cs[2 * e + 1] - a.y * sn[2 * e + 1]);
        }
      }
      // 8 channels = one 16-byte chunk of a swizzled row (c is a multiple of 8)
      *reinterpret_cast<uint4*>(sQ + swz_off(g, c, kDecQRows * 128)) = make_uint4(rlo[0], rlo[1], rlo[2], rlo[3]);
      *reinterpret_cast<uint4*>(sQ + swz_off(g, c + 64, kDecQRows * 128)) =
          make_uint4(rhi[0], rhi[1], rhi[2], rhi[3]);
      *reinterpret_cast<uint4*>(sQ + swz_off(16 + g, c, kDecQRows * 128)) = qlo;
      *reinterpret_cast<uint4*>(sQ + swz_off(16 + g, c + 64, kDecQRows * 128)) = qhi;
      // both P buffers start at zero (rows >= GROUP are never written)
      for (int e = tid; e < 2 * kDecHeads * 256 / 16; e += 128)
        reinterpret_cast<uint4*>(sP)[e] = make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_ready);
    }
    float m_run[GROUP], l_part[GROUP];
#pragma unroll
    for (int g = 0; g < GROUP; ++g) {
      m_run[g] = -INFINITY;
      l_part[g] = 0.f;
    }
    bool ok = true;
    for (int n = 0; n < n_tiles && ok; ++n) {
      if (!(ok = mbar_wait(&bars->s_full[n & 1], (n >> 1) & 1, abort))) break;
      if (wq == 0) JL_DTRACE_AT(n, 6);
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(t_lane + (n & 1) * 32, sr);
      const int j = c0 + n * kDecTile + tid;  // this thread's key
      const bool valid = j < c1;
      const bool rem = j <= jb;
      float sv[GROUP];
#pragma unroll
      for (int g = 0; g < GROUP; ++g)
        sv[g] = valid ? __uint_as_float(sr[rem ? g : 16 + g]) : -INFINITY;
      // per-head tile maximum over the 128 keys
      float* rb = red + (n & 1) * 64;
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        float x = sv[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
        if (lane == 0) rb[wq * 16 + g] = x;
      }
      mbar_arrive(&bars->red_full[n & 1]);
      if (!(ok = mbar_wait(&bars->red_full[n & 1], (n >> 1) & 1, abort))) break;
      if (wq == 0) JL_DTRACE_AT(n, 7);
      float alpha[GROUP];
      bool any_resc = false;
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        const float mt = fmaxf(fmaxf(rb[g], rb[16 + g]), fmaxf(rb[32 + g], rb[48 + g])) * sl2;
        const float m_new = fmaxf(m_run[g], mt);
        const bool resc = (m_run[g] != -INFINITY) && (m_new > m_run[g] + 8.f);
        alpha[g] = resc ? ex2_approx(m_run[g] - m_new) : 1.f;
        any_resc |= resc;
        if (resc || m_run[g] == -INFINITY) m_run[g] = m_new;
      }
      // PV(n-1) must be complete before P buffer (n & 1) is rewritten and before O is rescaled
      if (n > 0 && !(ok = mbar_wait(&bars->pv_done, (n - 1) & 1, abort))) break;
      if (wq == 0) JL_DTRACE_AT(n, 8);
      tc_fence_after();
      uint8_t* pb = sP + (n & 1) * (kDecHeads * 256);
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        const float m_use = (m_run[g] == -INFINITY) ? 0.f : m_run[g];
        const float pr = valid ? ex2_approx(fmaf(sv[g], sl2, -m_use)) : 0.f;
        l_part[g] = l_part[g] * alpha[g] + pr;
        *reinterpret_cast<uint16_t*>(pb + swz_off(g, tid, kDecHeads * 128)) = pack_bf16(pr);
      }
      if (any_resc && n > 0) {  // uniform: every thread computed the same alphas
        uint32_t o[32];
        tmem_ld32(t_lane + 64, o);  // columns 64..95; the first 16 are O^T
#pragma unroll
        for (int g = 0; g < GROUP; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
        tmem_st32(t_lane + 64, o);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_ready[n & 1]);
      if (wq == 0) JL_DTRACE_AT(n, 9);
    }
    // epilogue: row sums across the 128 threads, then the partial per query head
    if (ok && mbar_wait(&bars->pv_done, (n_tiles - 1) & 1, abort)) {
      tc_fence_after();
      float* rl = red + 128;  // [4][16]
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        float x = l_part[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (lane == 0) rl[wq * 16 + g] = x;
      }
      mbar_arrive(&bars->red_end);
      if (mbar_wait(&bars->red_end, 0, abort)) {
      uint32_t o[32];
      tmem_ld32(t_lane + 64, o);  // thread = channel tid
      float* ws = p.ws + ((static_cast<int64_t>(b) * p.n_split + split) * p.Hq + hk * ng) * (128 + 2);
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        if (g >= ng) break;
        float* dst = ws + static_cast<int64_t>(g) * (128 + 2);
        dst[2 + tid] = __uint_as_float(o[g]);
        if (tid == 0) {
          dst[0] = m_run[g];
          dst[1] = rl[g] + rl[16 + g] + rl[32 + g] + rl[48 + g];
        }
      }
      }
    }
    if (p.counters != nullptr) {
      // Every softmax thread, on every path (an aborted CTA takes a ticket too, so the
      // count completes): the arrival orders its partial stores before the ticket.
      mbar_arrive(&bars->fin);
      if (tid == 0) {
        mbar_wait_bounded(&bars->fin, 0);
        bars->last = take_ticket(p.counters + 2 * (b * p.Hkv + hk), p.epoch, n_active);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
  if (bars->last)  // uniform; set only with p.counters (the ticket acquired the other partials)
    merge_head_group(p, b, hk, ng, n_active, Lay::kThreads, false);
}

}  // namespace jl
