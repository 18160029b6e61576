// jl_append.cuh -- writing the base-RoPE KV cache the bifocal decode reads.
//
// Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
// RoPE", Methodology section 2: the KV cache stores the un-compressed base keys
// R(j) k_j at their exact absolute positions; the remote view is rebuilt on the
// fly at decode time, so the cache is written once per token and never again.
//
// jl_kv_fill_kernel     prompt tokens (packed varlen) -> cache entries
// jl_decode_append_kernel  one new token per entry: q~ = R(i) q, cache[i] = R(i) k, v
// jl_key_rotate_kernel  prompt keys -> the prefill's pre-rotated key rows (base and remote)
// The fill kernel gives each warp four (token, head) rows, the append kernel one;
// lanes own rotate-half pairs (c, c + D/2) and every access is a coalesced row read
// or write.
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
  int32_t w_pre;               // key rotation: w_pretrained, for G per sequence
  const float* cos_rem;        // key rotation, interpolation variant: remote rows rotate by
  const float* sin_rem;        // these tables at raw positions (NULL: R(f(j)))
  int64_t n_rem_rows;
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
// Each warp writes kFillRowsPerWarp consecutive (token, head) rows and issues all of
// their loads (key words, table entries, value words) before the first store, so a
// warp keeps several rows of DRAM reads in flight.  D = 128: lane l owns the
// rotate-half pairs (2l, 64+2l) and (2l+1, 64+2l+1), read as two bf16x2 words, and
// copies value channels 4l .. 4l+3 as one 8-byte word.  D = 64: lane l owns the pair
// (l, l+32) and value channels 2l, 2l+1.
constexpr int kFillRowsPerWarp = 4;

template <int D>
__global__ void __launch_bounds__(256) jl_kv_fill_kernel(const AppendParams p) {
  constexpr int R = kFillRowsPerWarp;
  constexpr int HALF = D / 2;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32 * R;
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = p.total_tokens * p.Hkv;
  int64_t src[R], dst[R], pos[R];
  bool live[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {  // locate each row and check it against the cache
    const int64_t row = row0 + r;
    live[r] = row < n_rows;
    src[r] = dst[r] = pos[r] = 0;
    if (!live[r]) continue;
    const int64_t t = row / p.Hkv;
    const int h = static_cast<int>(row % p.Hkv);
    int lo = 0, hi = p.batch - 1;  // sequence holding token t: last b with cu[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.lens[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    pos[r] = t - p.lens[b] + (p.past != nullptr ? p.past[b] : 0);
    const int64_t crow = (pos[r] < 0 || pos[r] >= p.cache_stride || pos[r] >= p.n_tab_rows) ? -1
                                                                                            : cache_row(p, b, pos[r]);
    if (crow < 0) {
      if (lane == 0) atomicOr(&g_status, kDevErrBounds);
      live[r] = false;
      continue;
    }
    src[r] = (t * p.Hkv + h) * D;
    dst[r] = (crow * p.Hkv + h) * D;
  }
  if constexpr (D == 128) {
    uint32_t ka[R], kb[R];
    float2 cs[R], sn[R];
    uint2 vw[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      ka[r] = *reinterpret_cast<const uint32_t*>(p.k + src[r] + 2 * lane);
      kb[r] = *reinterpret_cast<const uint32_t*>(p.k + src[r] + HALF + 2 * lane);
      cs[r] = *reinterpret_cast<const float2*>(p.cos_tab + pos[r] * HALF + 2 * lane);
      sn[r] = *reinterpret_cast<const float2*>(p.sin_tab + pos[r] * HALF + 2 * lane);
      vw[r] = *reinterpret_cast<const uint2*>(p.v + src[r] + 4 * lane);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ka[r]));
      const float2 bb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kb[r]));
      const float2 ya = make_float2(a.x * cs[r].x - bb.x * sn[r].x, a.y * cs[r].y - bb.y * sn[r].y);
      const float2 yb = make_float2(bb.x * cs[r].x + a.x * sn[r].x, bb.y * cs[r].y + a.y * sn[r].y);
      *reinterpret_cast<__nv_bfloat162*>(p.k_cache + dst[r] + 2 * lane) = __float22bfloat162_rn(ya);
      *reinterpret_cast<__nv_bfloat162*>(p.k_cache + dst[r] + HALF + 2 * lane) = __float22bfloat162_rn(yb);
      *reinterpret_cast<uint2*>(p.v_cache + dst[r] + 4 * lane) = vw[r];
    }
  } else {
    float ka[R], kb[R], cs[R], sn[R];
    uint32_t vw[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      ka[r] = __bfloat162float(p.k[src[r] + lane]);
      kb[r] = __bfloat162float(p.k[src[r] + HALF + lane]);
      cs[r] = p.cos_tab[pos[r] * HALF + lane];
      sn[r] = p.sin_tab[pos[r] * HALF + lane];
      vw[r] = *reinterpret_cast<const uint32_t*>(p.v + src[r] + 2 * lane);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      p.k_cache[dst[r] + lane] = __float2bfloat16_rn(ka[r] * cs[r] - kb[r] * sn[r]);
      p.k_cache[dst[r] + HALF + lane] = __float2bfloat16_rn(kb[r] * cs[r] + ka[r] * sn[r]);
      *reinterpret_cast<uint32_t*>(p.v_cache + dst[r] + 2 * lane) = vw[r];
    }
  }
}

// Keys for the bifocal prefill, rotated once before it instead of on every visit
// inside it ("Jet-Long", Methodology section 1: local pairs use the base positions,
// remote pairs the grouped positions f(x) = floor(x / G)).  Token t of sequence b sits
// at position j = t - cu_seqlens[b]; with G = max(1, ceil(L_b / w_pretrained)):
//   k_out[t]     = R(j) k_t          (local visits)
//   k_out[T + t] = R(floor(j / G)) k_t  (remote visits; not written for G = 1, whose
//                                       pairs are all local)
// For the interpolation variant (p.cos_rem set) the remote rows are rotated by the
// interpolated tables at the raw position j, for every sequence.
// Same lane layout and load batching as jl_kv_fill_kernel; p.k_cache is the output.
template <int D>
__global__ void __launch_bounds__(256) jl_key_rotate_kernel(const AppendParams p) {
  constexpr int R = kFillRowsPerWarp;
  constexpr int HALF = D / 2;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32 * R;
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = p.total_tokens * p.Hkv;
  const int64_t remote_off = p.total_tokens * p.Hkv * D;  // element offset of the remote rows
  const float* rcos = p.cos_rem != nullptr ? p.cos_rem : p.cos_tab;  // tables of the remote rows
  const float* rsin = p.sin_rem != nullptr ? p.sin_rem : p.sin_tab;
  int64_t src[R], pos[R], fpos[R];
  bool live[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {  // locate each row: its sequence, position and G
    const int64_t row = row0 + r;
    live[r] = row < n_rows;
    src[r] = pos[r] = 0;
    fpos[r] = -1;
    if (!live[r]) continue;
    const int64_t t = row / p.Hkv;
    const int h = static_cast<int>(row % p.Hkv);
    int lo = 0, hi = p.batch - 1;  // sequence holding token t: last b with cu[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.lens[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int L = p.lens[b + 1] - p.lens[b];
    const int G = max(1, (L + p.w_pre - 1) / p.w_pre);
    pos[r] = t - p.lens[b];
    if (pos[r] < 0 || pos[r] >= p.n_tab_rows) {  // the host checks max_seqlen <= n_tab_rows
      if (lane == 0) atomicOr(&g_status, kDevErrBounds);
      live[r] = false;
      continue;
    }
    if (p.cos_rem != nullptr) {
      if (pos[r] >= p.n_rem_rows) {  // the host checks max_seqlen <= n_rem_rows
        if (lane == 0) atomicOr(&g_status, kDevErrBounds);
        live[r] = false;
        continue;
      }
      fpos[r] = pos[r];
    } else if (G > 1) {
      fpos[r] = pos[r] / G;
    }
    src[r] = (t * p.Hkv + h) * D;
  }
  if constexpr (D == 128) {
    uint32_t ka[R], kb[R];
    float2 cs[R], sn[R], cf[R], sf[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      ka[r] = *reinterpret_cast<const uint32_t*>(p.k + src[r] + 2 * lane);
      kb[r] = *reinterpret_cast<const uint32_t*>(p.k + src[r] + HALF + 2 * lane);
      cs[r] = *reinterpret_cast<const float2*>(p.cos_tab + pos[r] * HALF + 2 * lane);
      sn[r] = *reinterpret_cast<const float2*>(p.sin_tab + pos[r] * HALF + 2 * lane);
      const int64_t fr = fpos[r] >= 0 ? fpos[r] : 0;
      cf[r] = *reinterpret_cast<const float2*>(rcos + fr * HALF + 2 * lane);
      sf[r] = *reinterpret_cast<const float2*>(rsin + fr * HALF + 2 * lane);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      const float2 a = unpack_bf16x2(ka[r]);
      const float2 bb = unpack_bf16x2(kb[r]);
      *reinterpret_cast<uint32_t*>(p.k_cache + src[r] + 2 * lane) =
          pack_bf16x2(a.x * cs[r].x - bb.x * sn[r].x, a.y * cs[r].y - bb.y * sn[r].y);
      *reinterpret_cast<uint32_t*>(p.k_cache + src[r] + HALF + 2 * lane) =
          pack_bf16x2(bb.x * cs[r].x + a.x * sn[r].x, bb.y * cs[r].y + a.y * sn[r].y);
      if (fpos[r] < 0) continue;
      *reinterpret_cast<uint32_t*>(p.k_cache + remote_off + src[r] + 2 * lane) =
          pack_bf16x2(a.x * cf[r].x - bb.x * sf[r].x, a.y * cf[r].y - bb.y * sf[r].y);
      *reinterpret_cast<uint32_t*>(p.k_cache + remote_off + src[r] + HALF + 2 * lane) =
          pack_bf16x2(bb.x * cf[r].x + a.x * sf[r].x, bb.y * cf[r].y + a.y * sf[r].y);
    }
  } else {
    float ka[R], kb[R], cs[R], sn[R], cf[R], sf[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      ka[r] = __bfloat162float(p.k[src[r] + lane]);
      kb[r] = __bfloat162float(p.k[src[r] + HALF + lane]);
      cs[r] = p.cos_tab[pos[r] * HALF + lane];
      sn[r] = p.sin_tab[pos[r] * HALF + lane];
      const int64_t fr = fpos[r] >= 0 ? fpos[r] : 0;
      cf[r] = rcos[fr * HALF + lane];
      sf[r] = rsin[fr * HALF + lane];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!live[r]) continue;
      p.k_cache[src[r] + lane] = __float2bfloat16_rn(ka[r] * cs[r] - kb[r] * sn[r]);
      p.k_cache[src[r] + HALF + lane] = __float2bfloat16_rn(kb[r] * cs[r] + ka[r] * sn[r]);
      if (fpos[r] < 0) continue;
      p.k_cache[remote_off + src[r] + lane] = __float2bfloat16_rn(ka[r] * cf[r] - kb[r] * sf[r]);
      p.k_cache[remote_off + src[r] + HALF + lane] = __float2bfloat16_rn(kb[r] * cf[r] + ka[r] * sf[r]);
    }
  }
}

// One decode step: entry b's new token sits at i = seqlens[b] - 1.  Rows 0..Hq-1
// rotate the query into q_out; rows Hq..Hq+Hkv-1 append key and value.
template <int D>
__global__ void __launch_bounds__(256) jl_decode_append_kernel(const AppendParams p) {
  griddep_launch_dependents();  // the decode that follows may launch now; it waits for this grid to finish
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
