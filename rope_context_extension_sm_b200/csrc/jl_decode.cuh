// jl_decode.cuh -- split-K single-query bifocal decode on a base-RoPE KV cache.
//
// Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
// RoPE", Methodology section 2, on-the-fly correction rotation: the cache keeps
// the un-compressed base keys k~_j = R(j) k_j at their absolute positions and is
// never rewritten; remote scores apply R(f(i) - i) to the active query and
// R(f(j) - j) to each cached key in registers, which rebuilds
// <R(f(i)) q, R(f(j)) k_j> because RoPE rotations compose additively.
//
// Grid (Hkv, n_split, B) -- the KV heads of one chunk run side by side; a CTA of 4 warps handles one KV head and one chunk of
// keys; each warp a quarter of the chunk.  Half-warps take one key each; lane r
// of a half-warp owns channels [r*H, r*H + H) and their rotate-half partners
// [D/2 + r*H, ...), so a key's correction stays inside the lane.  Scores are
// reduced with xor-shuffles, softmax is online per half-warp, and the four
// warps' states are merged in shared memory into one partial (m, l, o) per
// query head.  A second kernel merges the partials over the splits.
// Correction factors cos/sin(n_j theta), n_j = j - f(j), are formed by angle
// addition from table row n0 = n(first key of the chunk), held in registers,
// and row n_j - n0 < chunk: the rows 0..chunk-1 are shared by every CTA and
// stay cache-resident, so the correction adds no per-key HBM traffic.
#pragma once

#include "jl_device.cuh"

namespace jl {

constexpr int kDecodeThreads = 128;

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* seqlens;
  const float* cos_tab;
  const float* sin_tab;
  float* ws;              // partials [B][n_split][Hq][D + 2]
  __nv_bfloat16* out;
  float* lse;
  int64_t cache_stride;   // positions per batch entry
  int64_t n_tab_rows;     // rows of cos_tab / sin_tab
  const int32_t* block_table;  // paged caches: page of entry b's position j is block_table[b * max_pages + j / page_size]
  int32_t page_size, max_pages;
  int32_t Hq, Hkv, group;
  int32_t w0, w_pre, plain;
  int32_t chunk, n_split;
  float scale_log2;
  // Tensor-core decode only: two words per (entry, KV head) for the last-CTA merge
  // (null: jl_decode_combine_kernel merges), and this call's tag for those words.
  unsigned long long* counters;
  uint32_t epoch;
};

template <int H>
__device__ __forceinline__ void load_f32(const float* p, float (&x)[H]) {
  if constexpr (H == 4) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
  } else {
    const float2 u = *reinterpret_cast<const float2*>(p);
    x[0] = u.x; x[1] = u.y;
  }
}

template <int D>
__device__ __forceinline__ void load_half_bf16(const __nv_bfloat16* p, float (&x)[D / 32]) {
  if constexpr (D == 128) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = unpack_bf16x2(u.x);
    const float2 b = unpack_bf16x2(u.y);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    const float2 a = unpack_bf16x2(u);
    x[0] = a.x; x[1] = a.y;
  }
}

template <int D, int GROUP, bool PLAIN>
__global__ void __launch_bounds__(kDecodeThreads) jl_decode_split_kernel(const DecodeParams p) {
  constexpr int H = D / 32;  // channels per lane in each half
  constexpr int HALFD = D / 2;
  __shared__ float red_m[4][GROUP], red_l[4][GROUP];
  __shared__ float red_o[4][GROUP][D];

  const int hk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int ng = p.group;  // query heads of this KV head; GROUP is the capacity (rows >= ng stay zero)
  griddep_wait();              // inputs may come from the previous kernel (see jl_device.cuh)
  griddep_launch_dependents();
  const int L = p.seqlens[b];
  const int c0 = split * p.chunk;
  if (c0 >= L) return;
  if (status_failed()) return;
  const int c1 = min(c0 + p.chunk, L);
  const int i = L - 1;
  int G = 1, jb = -1;  // remote keys are j <= jb
  if (!PLAIN) {
    G = max(1, (L + p.w_pre - 1) / p.w_pre);
    if (G > 1) jb = i - p.w0;
  }
  const int n0 = c0 - c0 / G;  // correction index j - f(j) of the chunk's first key
  // the cache holds the length; the query's and the chunk's correction rows are in the table
  // (a key's row n0 + t is formed by angle addition from rows n0 and t, checked per key)
  JL_CHECK(L <= p.cache_stride && L <= p.n_split * p.chunk && (c1 - 1) - (c1 - 1) / G < p.n_tab_rows &&
           (i - i / G) < p.n_tab_rows && hk * ng + ng <= p.Hq);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = lane >> 4, r = lane & 15;
  const int cl = r * H;  // this lane's first channel in the low half
  const int per_warp = (c1 - c0 + 3) / 4;
  const int a0 = c0 + warp * per_warp;
  const int a1 = min(c1, a0 + per_warp);

  float m[GROUP], l[GROUP], o[GROUP][2 * H];
#pragma unroll
  for (int g = 0; g < GROUP; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 2 * H; ++e) o[g][e] = 0.f;
  }

  const int64_t row_stride = static_cast<int64_t>(p.Hkv) * D;
  const __nv_bfloat16* kbase = p.k + (static_cast<int64_t>(b) * p.cache_stride * p.Hkv + hk) * D;
  const __nv_bfloat16* vbase = p.v + (static_cast<int64_t>(b) * p.cache_stride * p.Hkv + hk) * D;

  // Two passes over this warp's keys: remote keys [a0, min(a1, jb+1)) then local keys.
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const bool remote = (pass == 0);
    const int s0 = remote ? a0 : max(a0, jb + 1);
    const int s1 = remote ? min(a1, jb + 1) : a1;
    if (s0 >= s1) continue;
    // row n0 of the correction factors (angle addition base), this lane's channels
    float ca[H], sa[H];
    if (remote) {
      load_f32<H>(p.cos_tab + static_cast<int64_t>(n0) * HALFD + cl, ca);
      load_f32<H>(p.sin_tab + static_cast<int64_t>(n0) * HALFD + cl, sa);
    }
    // query registers for this pass (scaled into log2 units)
    float qr[GROUP][2 * H];
#pragma unroll
    for (int g = 0; g < GROUP; ++g) {
      float lo[H], hi[H];
      if (g < ng) {
        const __nv_bfloat16* qp = p.q + (static_cast<int64_t>(b) * p.Hq + hk * ng + g) * D;
        load_half_bf16<D>(qp + cl, lo);
        load_half_bf16<D>(qp + HALFD + cl, hi);
      } else {
#pragma unroll
        for (int e = 0; e < H; ++e) lo[e] = hi[e] = 0.f;
      }
      if (remote) {  // R(f(i) - i) = R(-nq)
        const int64_t nq = i - i / G;
#pragma unroll
        for (int e = 0; e < H; ++e) {
          const float cs = p.cos_tab[nq * HALFD + cl + e], sn = p.sin_tab[nq * HALFD + cl + e];
          const float a = lo[e], bb = hi[e];
          lo[e] = a * cs + bb * sn;
          hi[e] = bb * cs - a * sn;
        }
      }
#pragma unroll
      for (int e = 0; e < H; ++e) {
        qr[g][e] = lo[e] * p.scale_log2;
        qr[g][H + e] = hi[e] * p.scale_log2;
      }
    }
#pragma unroll 2
    for (int j0 = s0; j0 < s1; j0 += 2) {
      const int j = j0 + kg;
      const bool valid = j < s1;
      const int jj = valid ? j : s0;
      float klo[H], khi[H], vlo[H], vhi[H];
      const __nv_bfloat16* kp = kbase + static_cast<int64_t>(jj) * row_stride;
      const __nv_bfloat16* vp = vbase + static_cast<int64_t>(jj) * row_stride;
      load_half_bf16<D>(kp + cl, klo);
      load_half_bf16<D>(kp + HALFD + cl, khi);
      load_half_bf16<D>(vp + cl, vlo);
      load_half_bf16<D>(vp + HALFD + cl, vhi);
      if (remote) {  // R(f(j) - j) = R(-n_j), n_j = n0 + t, t < chunk
        const int t = (jj - jj / G) - n0;
        JL_CHECK(t >= 0 && t < p.n_tab_rows);
        float cb[H], sb[H];
        load_f32<H>(p.cos_tab + static_cast<int64_t>(t) * HALFD + cl, cb);
        load_f32<H>(p.sin_tab + static_cast<int64_t>(t) * HALFD + cl, sb);
#pragma unroll
        for (int e = 0; e < H; ++e) {
          const float fc = ca[e] * cb[e] - sa[e] * sb[e];  // cos((n0 + t) theta)
          const float fs = sa[e] * cb[e] + ca[e] * sb[e];  // sin((n0 + t) theta)
          const float a = klo[e], bb = khi[e];
          klo[e] = a * fc + bb * fs;
          khi[e] = bb * fc - a * fs;
        }
      }
      float s[GROUP];
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < H; ++e) acc = fmaf(qr[g][e], klo[e], fmaf(qr[g][H + e], khi[e], acc));
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        s[g] = valid ? acc : -INFINITY;
      }
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        if (s[g] > m[g]) {
          const float alpha = ex2_approx(m[g] - s[g]);
          l[g] *= alpha;
#pragma unroll
          for (int e = 0; e < 2 * H; ++e) o[g][e] *= alpha;
          m[g] = s[g];
        }
        const float pr = ex2_approx(s[g] - m[g]);
        l[g] += (s[g] == -INFINITY) ? 0.f : pr;
        const float pv = (s[g] == -INFINITY) ? 0.f : pr;
#pragma unroll
        for (int e = 0; e < H; ++e) {
          o[g][e] = fmaf(pv, vlo[e], o[g][e]);
          o[g][H + e] = fmaf(pv, vhi[e], o[g][H + e]);
        }
      }
    }
  }

  // merge the two half-warps
#pragma unroll
  for (int g = 0; g < GROUP; ++g) {
    const float mo = __shfl_xor_sync(0xffffffffu, m[g], 16);
    const float mn = fmaxf(m[g], mo);
    const float sa = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - mn);
    const float sb = (mo == -INFINITY) ? 0.f : ex2_approx(mo - mn);
    const float lo_ = __shfl_xor_sync(0xffffffffu, l[g], 16);
    l[g] = l[g] * sa + lo_ * sb;
#pragma unroll
    for (int e = 0; e < 2 * H; ++e) {
      const float oo = __shfl_xor_sync(0xffffffffu, o[g][e], 16);
      o[g][e] = o[g][e] * sa + oo * sb;
    }
    m[g] = mn;
  }
  if (kg == 0) {
#pragma unroll
    for (int g = 0; g < GROUP; ++g) {
#pragma unroll
      for (int e = 0; e < H; ++e) {
        red_o[warp][g][cl + e] = o[g][e];
        red_o[warp][g][HALFD + cl + e] = o[g][H + e];
      }
      if (r == 0) {
        red_m[warp][g] = m[g];
        red_l[warp][g] = l[g];
      }
    }
  }
  __syncthreads();
  // merge the four warps: thread handles (g, c) pairs
  float* ws = p.ws + ((static_cast<int64_t>(b) * p.n_split + split) * p.Hq + hk * ng) * (D + 2);
  for (int idx = threadIdx.x; idx < ng * D; idx += kDecodeThreads) {
    const int g = idx / D, c = idx % D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, red_m[w][g]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float sc = (red_m[w][g] == -INFINITY) ? 0.f : ex2_approx(red_m[w][g] - mx);
      acc += red_o[w][g][c] * sc;
      lsum += red_l[w][g] * sc;
    }
    float* dst = ws + static_cast<int64_t>(g) * (D + 2);
    dst[2 + c] = acc;
    if (c == 0) {
      dst[0] = mx;
      dst[1] = lsum;
    }
  }
}

// Merge the per-split partials of one (batch entry, query head).  Phase 1: the
// block's maximum over the split maxima.  Phase 2: eight warps walk the splits
// (lane owns D/32 channels) with every load independent of the previous one;
// the warps' sums are added in shared memory.
constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) jl_decode_combine_kernel(const DecodeParams p) {
  constexpr int CPL = D / 32;  // channels per lane
  constexpr int NW = kCombineThreads / 32;
  const int qh = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();  // the next kernel may set itself up; it waits for this grid before reading
  griddep_wait();  // launched while the split kernel runs: its partials are complete from here on
  // The status word, the length and the first batch of partials are loaded together (one
  // round trip); splits past the length are masked once it is known.
  const unsigned status = *reinterpret_cast<volatile unsigned*>(&g_status);
  const int L = p.seqlens[b];
  const int ns = (L + p.chunk - 1) / p.chunk;
  const float* base = p.ws + (static_cast<int64_t>(b) * p.n_split * p.Hq + qh) * (D + 2);
  const int64_t sstride = static_cast<int64_t>(p.Hq) * (D + 2);
  __shared__ float sm_m[NW], sm_l[NW];
  __shared__ float sm_o[NW][D];
  // One pass: warp w blends splits w, w + NW, ... with a running maximum (their loads
  // all in flight together), then the warps' blends are joined in shared memory.
  constexpr int kBatch = 4;
  float M = -INFINITY, l = 0.f, acc[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
  for (int s0 = warp; s0 < p.n_split; s0 += kBatch * NW) {
    float ms[kBatch], ls[kBatch], os[kBatch][CPL];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {  // past n_split: split s0 again; past ns: masked below
      const int s = s0 + u * NW < p.n_split ? s0 + u * NW : s0;
      const float* ps = base + s * sstride;
      ms[u] = ps[0];
      ls[u] = ps[1];
#pragma unroll
      for (int e = 0; e < CPL; ++e) os[u][e] = ps[2 + lane * CPL + e];
    }
    if (s0 >= ns) break;
    bool valid[kBatch];
    float mb = M;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      valid[u] = s0 + u * NW < ns && ms[u] != -INFINITY;
      if (valid[u]) mb = fmaxf(mb, ms[u]);
    }
    if (mb == -INFINITY) continue;
    const float r = (M == -INFINITY) ? 0.f : ex2_approx(M - mb);
    l *= r;
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] *= r;
    M = mb;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (!valid[u]) continue;  // a stale split past the length may hold anything
      const float sc = ex2_approx(ms[u] - M);
      l = fmaf(ls[u], sc, l);
#pragma unroll
      for (int e = 0; e < CPL; ++e) acc[e] = fmaf(os[u][e], sc, acc[e]);
    }
  }
  JL_CHECK(L >= 1 && ns <= p.n_split);
#pragma unroll
  for (int e = 0; e < CPL; ++e) sm_o[warp][lane * CPL + e] = acc[e];
  if (lane == 0) {
    sm_m[warp] = M;
    sm_l[warp] = l;
  }
  __syncthreads();
  float Mx = sm_m[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) Mx = fmaxf(Mx, sm_m[w]);
  float sc[NW], lsum = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    sc[w] = (sm_m[w] == -INFINITY) ? 0.f : ex2_approx(sm_m[w] - Mx);
    lsum = fmaf(sm_l[w], sc[w], lsum);
  }
  // a split gave up: its partials are stale, so the output is marked undefined
  const bool bad = (status & kDevErrTimeout) != 0;
  const float nan = __int_as_float(0x7fc00000);
  for (int c = threadIdx.x; c < D; c += kCombineThreads) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) o = fmaf(sm_o[w][c], sc[w], o);
    p.out[(static_cast<int64_t>(b) * p.Hq + qh) * D + c] = __float2bfloat16_rn(bad ? nan : o / lsum);
    if (c == 0 && p.lse != nullptr)
      p.lse[static_cast<int64_t>(b) * p.Hq + qh] = bad ? nan : (Mx + log2f(lsum)) * 0.69314718055994531f;
  }
}

}  // namespace jl
