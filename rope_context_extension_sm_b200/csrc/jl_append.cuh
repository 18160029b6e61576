// jl_append.cuh -- writing the base-RoPE KV cache the bifocal decode reads.
//
// Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
// RoPE", Methodology section 2: the KV cache stores the un-compressed base keys
// R(j) k_j at their exact absolute positions; the remote view is rebuilt on the
// fly at decode time, so the cache is written once per token and never again.
//
// jl_kv_fill_kernel     prompt tokens (packed varlen) -> cache entries
// jl_decode_append_kernel  one new token per entry: q~ = R(i) q, cache[i] = R(i) k, v
// One warp per (token, head) row; lane l owns the rotate-half pairs (c, c + D/2)
// for c in [l*D/64, l*D/64 + D/64), loads are coalesced row reads.
#pragma once

#include "jl_device.cuh"

namespace jl {

constexpr unsigned kDevErrBounds = 2u;  // a position fell outside the cache

struct AppendParams {
  const __nv_bfloat16* q;      // decode: raw query rows [B][Hq][D]
  const __nv_bfloat16* k;      // raw key rows
  const __nv_bfloat16* v;
  const int32_t* lens;         // fill: cu_seqlens [batch+1]; decode: seqlens [B]
  const int32_t* past;         // fill: tokens already in each cache entry (NULL = 0)
  const float* cos_tab;
  const float* sin_tab;
  __nv_bfloat16* q_out;        // decode: rotated query rows
  __nv_bfloat16* k_cache;      // [B][stride][Hkv][D]
  __nv_bfloat16* v_cache;
  int64_t total_tokens;
  int64_t cache_stride;
  int64_t n_tab_rows;
  int32_t batch, Hq, Hkv;
  const int32_t* block_table;  // paged caches (NULL: contiguous [batch][cache_stride])
  int32_t page_size, max_pages, num_pages;
};

// Cache row of entry b's position pos (already checked against cache_stride):
// contiguous, or through the block table; -1 when the page index is outside the pool.
__device__ __forceinline__ int64_t cache_row(const AppendParams& p, int b, int64_t pos) {
  if (p.block_table == nullptr) return static_cast<int64_t>(b) * p.cache_stride + pos;
  const int32_t page = p.block_table[static_cast<int64_t>(b) * p.max_pages + pos / p.page_size];
  if (page < 0 || page >= p.num_pages) return -1;
  return static_cast<int64_t>(page) * p.page_size + pos % p.page_size;
}

// y = R(pos) x for one D-wide bf16 row, lane-parallel; writes y (and copies v_src -> v_dst if given).
template <int D>
__device__ __forceinline__ void rotate_row_global(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                                  int64_t pos, const AppendParams& p, int lane) {
  constexpr int HALF = D / 2;
  constexpr int PPL = D / 64;  // pairs per lane
#pragma unroll
  for (int e = 0; e < PPL; ++e) {
    const int c = lane * PPL + e;
    const float cs = p.cos_tab[pos * HALF + c], sn = p.sin_tab[pos * HALF + c];
    const float a = __bfloat162float(x[c]), b = __bfloat162float(x[c + HALF]);
    y[c] = __float2bfloat16_rn(a * cs - b * sn);
    y[c + HALF] = __float2bfloat16_rn(b * cs + a * sn);
  }
}

template <int D>
__device__ __forceinline__ void copy_row(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y, int lane) {
  constexpr int PER = D / 32;
#pragma unroll
  for (int e = 0; e < PER; ++e) y[lane * PER + e] = x[lane * PER + e];
}

// Prompt tokens: token t of sequence b sits at position past[b] + t - cu_seqlens[b].
template <int D>
__global__ void __launch_bounds__(256) jl_kv_fill_kernel(const AppendParams p) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;  // (token, head)
  const int lane = threadIdx.x & 31;
  if (row >= p.total_tokens * p.Hkv) return;
  const int64_t t = row / p.Hkv;
  const int h = static_cast<int>(row % p.Hkv);
  int lo = 0, hi = p.batch - 1;  // sequence holding token t: last b with cu[b] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.lens[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int64_t pos = t - p.lens[b] + (p.past != nullptr ? p.past[b] : 0);
  if (pos < 0 || pos >= p.cache_stride || pos >= p.n_tab_rows) {
    if (lane == 0) atomicOr(&g_status, kDevErrBounds);
    return;
  }
  const int64_t src = (t * p.Hkv + h) * D;
  const int64_t crow = cache_row(p, b, pos);
  if (crow < 0) {
    if (lane == 0) atomicOr(&g_status, kDevErrBounds);
    return;
  }
  const int64_t dst = (crow * p.Hkv + h) * D;
  rotate_row_global<D>(p.k + src, p.k_cache + dst, pos, p, lane);
  copy_row<D>(p.v + src, p.v_cache + dst, lane);
}

// One decode step: entry b's new token sits at i = seqlens[b] - 1.  Rows 0..Hq-1
// rotate the query into q_out; rows Hq..Hq+Hkv-1 append key and value.
template <int D>
__global__ void __launch_bounds__(256) jl_decode_append_kernel(const AppendParams p) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  const int per_b = p.Hq + p.Hkv;
  if (row >= static_cast<int64_t>(p.batch) * per_b) return;
  const int b = static_cast<int>(row / per_b), r = static_cast<int>(row % per_b);
  const int64_t i = static_cast<int64_t>(p.lens[b]) - 1;
  if (i < 0 || i >= p.cache_stride || i >= p.n_tab_rows) {
    if (lane == 0) atomicOr(&g_status, kDevErrBounds);
    return;
  }
  if (r < p.Hq) {
    const int64_t o = (static_cast<int64_t>(b) * p.Hq + r) * D;
    rotate_row_global<D>(p.q + o, p.q_out + o, i, p, lane);
  } else {
    const int h = r - p.Hq;
    const int64_t src = (static_cast<int64_t>(b) * p.Hkv + h) * D;
    const int64_t crow = cache_row(p, b, i);
    if (crow < 0) {
      if (lane == 0) atomicOr(&g_status, kDevErrBounds);
      return;
    }
    const int64_t dst = (crow * p.Hkv + h) * D;
    rotate_row_global<D>(p.k + src, p.k_cache + dst, i, p, lane);
    copy_row<D>(p.v + src, p.v_cache + dst, lane);
  }
}

}  // namespace jl
