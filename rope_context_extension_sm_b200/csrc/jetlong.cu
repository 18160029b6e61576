// jetlong.cu -- the C ABI of libjetlong.so (declared in include/jetlong.h):
// argument validation, TMA tensor-map encoding and kernel launches for the
// bifocal prefill, the split-K bifocal decode, their plain comparators and the
// RoPE tables.  One translation unit, so the device status word needs no
// relocatable device code.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "jetlong.h"
#include "jl_append.cuh"
#include "jl_decode.cuh"
#include "jl_decode_tc.cuh"
#include "jl_prefill.cuh"
#include "jl_tables.cuh"

namespace {

thread_local std::string g_err;

jl_status fail(jl_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
jl_status fail(jl_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

jl_status ok() {
  g_err.clear();
  return JL_OK;
}

jl_status cuda_fail(cudaError_t e, const char* what) {
  return fail(JL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------ kernel attributes --
//
// Function attributes (the dynamic shared-memory limit) belong to the device
// context a launch runs in, so the one-time setting is kept per (device,
// kernel): a process that drives a second GPU sets it there too.  A failed
// attempt is not remembered, so the next launch tries again.

struct KernelAttr {
  cudaError_t err;
  int regs;  // registers per thread of the built kernel
};

std::mutex g_attr_mu;
std::map<std::pair<int, const void*>, KernelAttr> g_attr;

KernelAttr kernel_attr(const void* kern, int smem_bytes) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return {e, 0};
  std::lock_guard<std::mutex> lock(g_attr_mu);
  const auto key = std::make_pair(dev, kern);
  const auto it = g_attr.find(key);
  if (it != g_attr.end()) return it->second;
  KernelAttr a{cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes), 0};
  if (a.err == cudaSuccess) {
    cudaFuncAttributes fa{};
    a.err = cudaFuncGetAttributes(&fa, kern);
    a.regs = fa.numRegs;
  }
  if (a.err == cudaSuccess) g_attr[key] = a;
  return a;
}

// ---------------------------------------------------------------- TMA maps --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [tokens][heads][d] bf16, box = 64 channels x 1 head x 128 tokens, 128B swizzle.
jl_status make_map(CUtensorMap* map, const void* base, int64_t tokens, int heads, int d) {
  auto fn = encode_fn();
  if (!fn) return fail(JL_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(heads) * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(JL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return JL_OK;
}

// Launch with the programmatic stream-serialization attribute: the kernel may be
// scheduled while the previous kernel of the stream still runs, and waits for it
// in griddep_wait() (jl_device.cuh) before touching its results.  This hides the
// launch latency of the short decode kernels behind the kernel before them.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ----------------------------------------------------------------- prefill --

template <int D, int NQT>
jl_status launch_prefill(const void* q, const void* k, const void* v, const jl::PrefillParams& prm,
                         cudaStream_t st) {
  using Lay = jl::PrefillLayout<D, NQT>;
  CUtensorMap tq, tk, tv;
  jl_status s;
  if ((s = make_map(&tq, q, prm.total_tokens, prm.Hq, D)) != JL_OK) return s;
  // keys/values: the packed prompt, or (chunked prefill) the base-RoPE caches; pre-rotated
  // keys hold a base and a remote row per token
  const int64_t kv_rows = prm.cached ? static_cast<int64_t>(prm.batch) * prm.cache_stride : prm.total_tokens;
  if ((s = make_map(&tk, k, prm.krot ? 2 * prm.total_tokens : kv_rows, prm.Hkv, D)) != JL_OK) return s;
  if ((s = make_map(&tv, v, kv_rows, prm.Hkv, D)) != JL_OK) return s;
  auto kern = jl::jl_prefill_kernel<D, NQT>;
  const KernelAttr attr = kernel_attr(reinterpret_cast<const void*>(kern), Lay::kAlloc);
  if (attr.err != cudaSuccess) return cuda_fail(attr.err, "cudaFuncSetAttribute(prefill)");
  const int launch_regs = attr.regs;
  // The kernel moves registers between its warpgroups (setmaxnreg); the softmax
  // warpgroups' increase would wait forever if the launch allocation could not
  // cover the split, so such a build is refused here rather than launched.
  if (Lay::kSplitRegs && static_cast<int64_t>(launch_regs) * Lay::kThreads < Lay::kRegsNeeded)
    return fail(JL_ERR_UNSUPPORTED, "prefill kernel built with %d registers per thread; the register split needs %u",
                launch_regs, Lay::kRegsLaunch);
  const int64_t blocks = static_cast<int64_t>(prm.n_qtiles) * prm.batch * prm.Hkv * prm.slots;
  if (blocks > 0x7fffffff) return fail(JL_ERR_UNSUPPORTED, "prefill grid too large (%lld blocks)", (long long)blocks);
  kern<<<static_cast<unsigned>(blocks), Lay::kThreads, Lay::kAlloc, st>>>(tq, tk, tv, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return ok();
}

// Validates and fills the kernel parameters; returns JL_OK with *empty set when
// there is nothing to compute.
jl_status prefill_params(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                         int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                         int32_t w0, int32_t w_pretrained, int plain, const float* cos_tab, const float* sin_tab,
                         int64_t n_tab_rows, float softmax_scale, void* out, float* lse, jl::PrefillParams* prm,
                         bool* empty) {
  *empty = false;
  if (batch < 0) return fail(JL_ERR_INVALID, "batch must be >= 0 (got %d)", batch);
  if (total_tokens < 0 || total_tokens > 0x7fffffffLL)
    return fail(JL_ERR_INVALID, "total_tokens must be in [0, 2^31) (got %lld)", (long long)total_tokens);
  if (max_seqlen < 0) return fail(JL_ERR_INVALID, "max_seqlen must be >= 0 (got %d)", max_seqlen);
  if (head_dim != 64 && head_dim != 128)
    return fail(JL_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(JL_ERR_INVALID, "need Hq >= 1, Hkv >= 1 and Hq %% Hkv == 0 (got Hq=%d, Hkv=%d)", Hq, Hkv);
  if (w0 < 0) return fail(JL_ERR_INVALID, "w0 must be >= 0 (got %d)", w0);
  if (w_pretrained < 1) return fail(JL_ERR_INVALID, "w_pretrained must be >= 1 (got %d)", w_pretrained);
  if (batch == 0 || total_tokens == 0 || max_seqlen == 0) {
    *empty = true;
    return ok();
  }
  if (!q || !k || !v || !cu_seqlens || !cos_tab || !sin_tab || !out)
    return fail(JL_ERR_INVALID, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cos_tab) ||
      !aligned16(sin_tab))
    return fail(JL_ERR_INVALID, "q, k, v, out and the tables must be 16-byte aligned");
  if (n_tab_rows < max_seqlen)
    return fail(JL_ERR_INVALID, "n_tab_rows (%lld) must be >= max_seqlen (%d)", (long long)n_tab_rows, max_seqlen);
  *prm = jl::PrefillParams{};
  prm->cu_seqlens = cu_seqlens;
  prm->cos_tab = cos_tab;
  prm->sin_tab = sin_tab;
  prm->out = static_cast<__nv_bfloat16*>(out);
  prm->lse = lse;
  prm->total_tokens = total_tokens;
  prm->n_tab_rows = n_tab_rows;
  prm->batch = batch;
  prm->n_qtiles = (max_seqlen + jl::kBM - 1) / jl::kBM;
  prm->Hq = Hq;
  prm->Hkv = Hkv;
  prm->group = Hq / Hkv;
  prm->w0 = w0;
  prm->w_pre = w_pretrained;
  prm->plain = plain;
  prm->mode = 0;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  prm->scale_log2 = scale * 1.4426950408889634f;
  prm->slots = prm->group / ((prm->group % 2) == 0 ? 2 : 1);
  return ok();
}

// One query head per CTA with double-buffered scores (jl_prefill_db_kernel).
template <int D>
jl_status launch_prefill_db(const void* q, const void* k, const void* v, jl::PrefillParams prm, cudaStream_t st) {
  using Lay = jl::PrefillDbLayout<D>;
  prm.slots = prm.group;  // every query head is its own CTA
  CUtensorMap tq, tk, tv;
  jl_status s;
  if ((s = make_map(&tq, q, prm.total_tokens, prm.Hq, D)) != JL_OK) return s;
  const int64_t kv_rows = prm.cached ? static_cast<int64_t>(prm.batch) * prm.cache_stride : prm.total_tokens;
  if ((s = make_map(&tk, k, prm.krot ? 2 * prm.total_tokens : kv_rows, prm.Hkv, D)) != JL_OK) return s;
  if ((s = make_map(&tv, v, kv_rows, prm.Hkv, D)) != JL_OK) return s;
  auto kern = jl::jl_prefill_db_kernel<D>;
  const KernelAttr attr = kernel_attr(reinterpret_cast<const void*>(kern), Lay::kAlloc);
  if (attr.err != cudaSuccess) return cuda_fail(attr.err, "cudaFuncSetAttribute(prefill)");
  // the softmax warpgroup's register increase would wait forever if the launch
  // allocation could not cover the split, so such a build is refused
  if (static_cast<int64_t>(attr.regs) * Lay::kThreads < Lay::kRegsNeeded)
    return fail(JL_ERR_UNSUPPORTED, "prefill kernel built with %d registers per thread; the register split needs %u",
                attr.regs, Lay::kRegsLaunch);
  const int64_t blocks = static_cast<int64_t>(prm.n_qtiles) * prm.batch * prm.Hkv * prm.slots;
  if (blocks > 0x7fffffff) return fail(JL_ERR_UNSUPPORTED, "prefill grid too large (%lld blocks)", (long long)blocks);
  kern<<<static_cast<unsigned>(blocks), Lay::kThreads, Lay::kAlloc, st>>>(tq, tk, tv, prm);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return ok();
}

// Which kernel: an even GQA group pairs two query heads per CTA (jl_prefill_kernel
// <D, 2>: one K/V tile and one rotation serve both).  An odd group (multi-head
// attention included) has a head with no partner; at head_dim 128 it runs one head
// per CTA with double-buffered scores (jl_prefill_db_kernel), about 1.3x the
// single-buffered one-head kernel on those shapes.  JL_PREFILL_DB = 1 at build time
// sends every head_dim-128 call there (for measurements).
#ifndef JL_PREFILL_DB
#define JL_PREFILL_DB 0
#endif

jl_status launch_prefill_any(const void* q, const void* k, const void* v, const jl::PrefillParams& prm,
                             int32_t head_dim, cudaStream_t st) {
  const bool pair = (prm.group % 2) == 0;
  if (head_dim == 128 && (JL_PREFILL_DB || !pair)) return launch_prefill_db<128>(q, k, v, prm, st);
  if (head_dim == 128)
    return pair ? launch_prefill<128, 2>(q, k, v, prm, st) : launch_prefill<128, 1>(q, k, v, prm, st);
  return pair ? launch_prefill<64, 2>(q, k, v, prm, st) : launch_prefill<64, 1>(q, k, v, prm, st);
}

// Bytes of the pre-rotated keys: a base row R(j) k and a remote row R(f(j)) k per
// token and KV head.
size_t key_rot_bytes(int64_t total_tokens, int32_t Hkv, int32_t head_dim) {
  if (total_tokens <= 0 || Hkv <= 0 || head_dim <= 0) return 0;
  return 2 * static_cast<size_t>(total_tokens) * Hkv * head_dim * sizeof(__nv_bfloat16);
}

// Rotates the prompt keys once into the workspace (jl_key_rotate_kernel): base rows
// R(j) k, then remote rows R(f(j)) k (w_pre gives G per sequence), or with cos_rem the
// interpolated rotation at the raw position.
jl_status rotate_keys(const void* k, const int32_t* cu_seqlens, int32_t batch, int64_t total_tokens, int32_t Hkv,
                      int32_t head_dim, int32_t w_pre, const float* cos_tab, const float* sin_tab,
                      int64_t n_tab_rows, const float* cos_rem, const float* sin_rem, int64_t n_rem_rows,
                      void* workspace, size_t workspace_bytes, cudaStream_t st) {
  const size_t need = key_rot_bytes(total_tokens, Hkv, head_dim);
  if (workspace_bytes < need)
    return fail(JL_ERR_INVALID, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(JL_ERR_INVALID, "the workspace must be 16-byte aligned");
  if (total_tokens >= (int64_t(1) << 30))  // the remote rows sit total_tokens rows on, as int32 TMA coordinates
    return fail(JL_ERR_UNSUPPORTED, "a key workspace needs total_tokens < 2^30 (got %lld)", (long long)total_tokens);
  jl::AppendParams ap{};
  ap.k = static_cast<const __nv_bfloat16*>(k);
  ap.lens = cu_seqlens;
  ap.cos_tab = cos_tab;
  ap.sin_tab = sin_tab;
  ap.k_cache = static_cast<__nv_bfloat16*>(workspace);
  ap.total_tokens = total_tokens;
  ap.n_tab_rows = n_tab_rows;
  ap.batch = batch;
  ap.Hkv = Hkv;
  ap.w_pre = w_pre;
  ap.cos_rem = cos_rem;
  ap.sin_rem = sin_rem;
  ap.n_rem_rows = n_rem_rows;
  const int64_t warps = (total_tokens * Hkv + jl::kFillRowsPerWarp - 1) / jl::kFillRowsPerWarp;
  const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
  if (head_dim == 128) jl::jl_key_rotate_kernel<128><<<blocks, 256, 0, st>>>(ap);
  else jl::jl_key_rotate_kernel<64><<<blocks, 256, 0, st>>>(ap);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "key rotation launch");
  return ok();
}

// With a workspace, the keys are rotated once into it (jl_key_rotate_kernel) and the
// prefill kernel reads them as they are; without one, its rotation warps rotate every
// key tile on every visit.
jl_status prefill_common(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                         int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                         int32_t w0, int32_t w_pretrained, int plain, const float* cos_tab, const float* sin_tab,
                         int64_t n_tab_rows, float softmax_scale, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, cudaStream_t st) {
  jl::PrefillParams prm;
  bool empty;
  jl_status s = prefill_params(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, w0,
                               w_pretrained, plain, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, &prm,
                               &empty);
  if (s != JL_OK || empty) return s;
  if (workspace == nullptr) return launch_prefill_any(q, k, v, prm, head_dim, st);
  // plain: every pair is local, so no remote rows (G = 1 for every length below 2^30,
  // which rotate_keys requires, without overflowing L + w_pre - 1 in int32)
  if ((s = rotate_keys(k, cu_seqlens, batch, total_tokens, Hkv, head_dim, plain ? (1 << 30) : w_pretrained,
                       cos_tab, sin_tab, n_tab_rows, nullptr, nullptr, 0, workspace, workspace_bytes, st)) != JL_OK)
    return s;
  prm.krot = 1;
  return launch_prefill_any(q, workspace, v, prm, head_dim, st);
}

size_t three_pass_ws_bytes(int64_t total_tokens, int32_t Hq, int32_t head_dim) {
  if (total_tokens <= 0 || Hq <= 0 || head_dim <= 0) return 0;
  return 3 * static_cast<size_t>(total_tokens) * Hq * head_dim * 4 + 3 * static_cast<size_t>(total_tokens) * Hq * 4;
}

// ------------------------------------------------------------------ decode --

// Tensor-core decode (head_dim 128) splits the keys in chunks of whole 128-key
// tiles, sized for one wave of CTAs; head_dim 64 uses the CUDA-core split kernel.
// Both take up to 16 query heads per KV head: each is built for the group
// capacities 1, 2, 4, 8 and 16, and a group in between runs in the next capacity
// up with the spare query rows held at zero.
constexpr int32_t kMaxDecodeGroup = 16;
bool decode_uses_tc(int32_t head_dim, int32_t Hq, int32_t Hkv) {
  return head_dim == 128 && Hq / Hkv <= kMaxDecodeGroup;
}

// Keys per split.  CUDA-core kernel: a power of two in [64, 512].  Tensor-core
// kernel: whole 128-key tiles, as many splits per (entry, KV head) as fit the
// 148 SMs of a B200 in ONE wave (one CTA per SM): a CTA left over for a second
// wave would run after all the others and set the kernel's time.  When one wave
// would leave each CTA more than kMaxTilesPerSplit tiles to walk (many entries x
// KV heads), the splits are cut to that length instead and the grid runs in
// several waves; splits past an entry's length exit at once.
constexpr int64_t kSMs = 148;
constexpr int64_t kMaxTilesPerSplit = 128;

int chunk_cuda_core(int32_t max_seqlen) {
  int c = 64;
  while (c < 512 && static_cast<int64_t>(c) * 256 < max_seqlen) c *= 2;
  return c;
}

int chunk_tc(int32_t B, int32_t Hkv, int32_t max_seqlen) {
  const int64_t tiles = (static_cast<int64_t>(max_seqlen) + jl::kDecTile - 1) / jl::kDecTile;
  const int64_t ctas_per_split = static_cast<int64_t>(Hkv) * B;
  const int64_t n_target = std::max<int64_t>(1, kSMs / std::max<int64_t>(1, ctas_per_split));
  const int64_t per = std::min(kMaxTilesPerSplit, std::max<int64_t>(1, (tiles + n_target - 1) / n_target));
  return static_cast<int>(per * jl::kDecTile);
}

template <int GROUP, bool PLAIN>
jl_status launch_decode_tc(const jl::DecodeParams& prm, int B, cudaStream_t st) {
  using Lay = jl::DecTcLayout<GROUP>;
  CUtensorMap tk, tv;
  jl_status s;
  // contiguous caches, or (paged) the page pool; the kernel bounds every page it reads
  const int64_t rows = prm.block_table != nullptr ? prm.cache_stride : static_cast<int64_t>(B) * prm.cache_stride;
  if ((s = make_map(&tk, prm.k, rows, prm.Hkv, 128)) != JL_OK) return s;
  if ((s = make_map(&tv, prm.v, rows, prm.Hkv, 128)) != JL_OK) return s;
  auto kern = jl::jl_decode_tc_kernel<GROUP, PLAIN>;
  const KernelAttr attr = kernel_attr(reinterpret_cast<const void*>(kern), Lay::kAlloc);
  if (attr.err != cudaSuccess) return cuda_fail(attr.err, "cudaFuncSetAttribute(decode)");
  dim3 grid(prm.Hkv, prm.n_split, B);
  cudaError_t e = launch_pdl(kern, grid, dim3(Lay::kThreads), Lay::kAlloc, st, tk, tv, prm);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  if (prm.counters == nullptr) {  // no merge counters: a second kernel merges the splits
    e = launch_pdl(jl::jl_decode_combine_kernel<128>, dim3(prm.Hq, B), dim3(jl::kCombineThreads), 0, st, prm);
    if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  }
  return ok();
}

template <int D, int GROUP, bool PLAIN>
jl_status launch_decode(const jl::DecodeParams& prm, int B, cudaStream_t st) {
  dim3 grid(prm.Hkv, prm.n_split, B);
  cudaError_t e = launch_pdl(jl::jl_decode_split_kernel<D, GROUP, PLAIN>, grid, dim3(jl::kDecodeThreads), 0, st, prm);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  e = launch_pdl(jl::jl_decode_combine_kernel<D>, dim3(prm.Hq, B), dim3(jl::kCombineThreads), 0, st, prm);
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return ok();
}

template <int D, bool PLAIN>
jl_status dispatch_group(const jl::DecodeParams& prm, int B, cudaStream_t st) {
  const int g = prm.group;
  if (g < 1 || g > kMaxDecodeGroup)
    return fail(JL_ERR_UNSUPPORTED, "decode supports 1 to %d query heads per KV head (got %d)", kMaxDecodeGroup, g);
  if constexpr (D == 128) {  // tensor cores
    if (g <= 1) return launch_decode_tc<1, PLAIN>(prm, B, st);
    if (g <= 2) return launch_decode_tc<2, PLAIN>(prm, B, st);
    if (g <= 4) return launch_decode_tc<4, PLAIN>(prm, B, st);
    if (g <= 8) return launch_decode_tc<8, PLAIN>(prm, B, st);
    return launch_decode_tc<16, PLAIN>(prm, B, st);
  } else {  // head_dim 64: CUDA cores
    if (g <= 1) return launch_decode<D, 1, PLAIN>(prm, B, st);
    if (g <= 2) return launch_decode<D, 2, PLAIN>(prm, B, st);
    if (g <= 4) return launch_decode<D, 4, PLAIN>(prm, B, st);
    if (g <= 8) return launch_decode<D, 8, PLAIN>(prm, B, st);
    return launch_decode<D, 16, PLAIN>(prm, B, st);
  }
}

// Workspace: the split partials [B][n_split][Hq][head_dim + 2] floats, then (from a
// 256-byte boundary) two 8-byte merge counter words per (entry, KV head), B * Hq
// pairs at most.
size_t partials_bytes(int32_t B, int32_t Hq, int32_t head_dim, int32_t max_seqlen, int chunk) {
  const int64_t n_split = (max_seqlen + chunk - 1) / chunk;
  const size_t n = static_cast<size_t>(B) * n_split * Hq * (head_dim + 2) * sizeof(float);
  return (n + 255) / 256 * 256;
}

size_t ws_bytes_for(int32_t B, int32_t Hq, int32_t head_dim, int32_t max_seqlen, int chunk) {
  return partials_bytes(B, Hq, head_dim, max_seqlen, chunk) + static_cast<size_t>(B) * Hq * 2 * sizeof(uint64_t);
}

// The head_dim-128 decode merges the split partials in a second kernel unless built
// with JL_DECODE_LAST_CTA_MERGE = 1, where the last split CTA of each (entry, KV head)
// merges them in the same launch (measured slower on B200, kept as a tested variant).
#ifndef JL_DECODE_LAST_CTA_MERGE
#define JL_DECODE_LAST_CTA_MERGE 0
#endif

// Tag of one decode call for its merge counters (never 0, the tag of a cleared
// word).  Successive calls get distinct tags for 2^32 - 1 calls.
uint32_t next_decode_tag() {
  static std::atomic<uint32_t> tag{0x5bd1e995u};
  uint32_t t = tag.fetch_add(1u, std::memory_order_relaxed) + 1u;
  return t != 0u ? t : tag.fetch_add(1u, std::memory_order_relaxed) + 1u;
}

// Upper bound over both decode kernels and every KV-head count the query heads
// allow (the query does not know Hkv, which picks the kernel and the split).
size_t decode_ws_bytes(int32_t B, int32_t Hq, int32_t head_dim, int32_t max_seqlen) {
  if (B <= 0 || Hq <= 0 || head_dim <= 0 || max_seqlen <= 0) return 0;
  size_t n = ws_bytes_for(B, Hq, head_dim, max_seqlen, chunk_cuda_core(max_seqlen));
  for (int32_t hkv = 1; hkv <= Hq; ++hkv) {
    if (Hq % hkv != 0 || !decode_uses_tc(head_dim, Hq, hkv)) continue;
    const size_t t = ws_bytes_for(B, Hq, head_dim, max_seqlen, chunk_tc(B, hkv, max_seqlen));
    n = t > n ? t : n;
  }
  return n;
}

jl_status decode_common(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, int32_t B,
                        int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                        int32_t w0, int32_t w_pretrained, int plain, const float* cos_tab, const float* sin_tab,
                        int64_t n_tab_rows, float softmax_scale, void* out, float* lse, void* workspace,
                        size_t workspace_bytes, cudaStream_t st, const int32_t* block_table = nullptr,
                        int32_t page_size = 0, int32_t max_pages = 0) {
  if (B < 0) return fail(JL_ERR_INVALID, "B must be >= 0 (got %d)", B);
  if (head_dim != 64 && head_dim != 128)
    return fail(JL_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(JL_ERR_INVALID, "need Hq >= 1, Hkv >= 1 and Hq %% Hkv == 0 (got Hq=%d, Hkv=%d)", Hq, Hkv);
  if (w0 < 0) return fail(JL_ERR_INVALID, "w0 must be >= 0 (got %d)", w0);
  if (w_pretrained < 1) return fail(JL_ERR_INVALID, "w_pretrained must be >= 1 (got %d)", w_pretrained);
  if (B == 0) return ok();
  if (max_seqlen < 1) return fail(JL_ERR_INVALID, "max_seqlen must be >= 1 (got %d)", max_seqlen);
  if (cache_stride < max_seqlen)
    return fail(JL_ERR_INVALID, "cache_stride (%lld) must be >= max_seqlen (%d)", (long long)cache_stride,
                max_seqlen);
  if (n_tab_rows < max_seqlen)
    return fail(JL_ERR_INVALID, "n_tab_rows (%lld) must be >= max_seqlen (%d)", (long long)n_tab_rows, max_seqlen);
  if (block_table == nullptr && static_cast<int64_t>(B) * cache_stride > 0x7fffffffLL)
    return fail(JL_ERR_UNSUPPORTED, "B * cache_stride must be < 2^31 (got %lld)", (long long)B * cache_stride);
  if (!q || !k_cache || !v_cache || !seqlens || !cos_tab || !sin_tab || !out || !workspace)
    return fail(JL_ERR_INVALID, "null pointer argument");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace) ||
      !aligned16(cos_tab) || !aligned16(sin_tab))
    return fail(JL_ERR_INVALID, "q, caches, out, workspace and the tables must be 16-byte aligned");
  const size_t need = decode_ws_bytes(B, Hq, head_dim, max_seqlen);
  if (workspace_bytes < need)
    return fail(JL_ERR_INVALID, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  jl::DecodeParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k_cache);
  prm.v = static_cast<const __nv_bfloat16*>(v_cache);
  prm.seqlens = seqlens;
  prm.cos_tab = cos_tab;
  prm.sin_tab = sin_tab;
  prm.ws = static_cast<float*>(workspace);
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.cache_stride = cache_stride;  // paged: rows of the page pool
  prm.n_tab_rows = n_tab_rows;
  prm.block_table = block_table;
  prm.page_size = page_size;
  prm.max_pages = max_pages;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.w0 = w0;
  prm.w_pre = w_pretrained;
  prm.plain = plain;
  const bool tc = decode_uses_tc(head_dim, Hq, Hkv);
  prm.chunk = tc ? chunk_tc(B, Hkv, max_seqlen) : chunk_cuda_core(max_seqlen);
  prm.n_split = (max_seqlen + prm.chunk - 1) / prm.chunk;
  if (tc && JL_DECODE_LAST_CTA_MERGE) {  // the tensor-core kernel merges in its last CTA per (entry, KV head)
    prm.counters = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) +
                                                         partials_bytes(B, Hq, head_dim, max_seqlen, prm.chunk));
    prm.epoch = next_decode_tag();
  }
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  prm.scale_log2 = scale * 1.4426950408889634f;
  if (head_dim == 128)
    return plain ? dispatch_group<128, true>(prm, B, st) : dispatch_group<128, false>(prm, B, st);
  return plain ? dispatch_group<64, true>(prm, B, st) : dispatch_group<64, false>(prm, B, st);
}

// ------------------------------------------------------------ cache writers --

// fill = true: prompt tokens (packed by lens = cu_seqlens, optional past offsets);
// fill = false: one decode token per entry (lens = seqlens), query rotated to q_out.
jl_status append_common(const void* q, const void* k, const void* v, const int32_t* lens, const int32_t* past,
                        int32_t batch, int64_t total_tokens, int32_t Hq, int32_t Hkv, int32_t head_dim,
                        const float* cos_tab, const float* sin_tab, int64_t n_tab_rows, void* q_out, void* k_cache,
                        void* v_cache, int64_t cache_stride, const int32_t* block_table, int32_t page_size,
                        int32_t max_pages, int32_t num_pages, cudaStream_t st, bool fill) {
  if (batch < 0 || total_tokens < 0 || Hkv < 1 || cache_stride < 1 || n_tab_rows < 1 || (!fill && Hq < 1))
    return fail(JL_ERR_INVALID, "need batch >= 0, tokens >= 0, heads >= 1, cache_stride >= 1, n_tab_rows >= 1");
  if (head_dim != 64 && head_dim != 128)
    return fail(JL_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (batch == 0 || (fill && total_tokens == 0)) return ok();
  if (!k || !v || !lens || !cos_tab || !sin_tab || !k_cache || !v_cache || (!fill && (!q || !q_out)))
    return fail(JL_ERR_INVALID, "null pointer argument");
  jl::AppendParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k);
  prm.v = static_cast<const __nv_bfloat16*>(v);
  prm.lens = lens;
  prm.past = past;
  prm.cos_tab = cos_tab;
  prm.sin_tab = sin_tab;
  prm.q_out = static_cast<__nv_bfloat16*>(q_out);
  prm.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  prm.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  prm.total_tokens = total_tokens;
  prm.cache_stride = cache_stride;  // paged: positions one entry can hold (max_pages * page_size)
  prm.n_tab_rows = n_tab_rows;
  prm.batch = batch;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.block_table = block_table;
  prm.page_size = page_size;
  prm.max_pages = max_pages;
  prm.num_pages = num_pages;
  const int64_t rows = fill ? total_tokens * Hkv : static_cast<int64_t>(batch) * (Hq + Hkv);
  const int64_t warps = fill ? (rows + jl::kFillRowsPerWarp - 1) / jl::kFillRowsPerWarp : rows;
  const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
  if (fill) {
    if (head_dim == 128) jl::jl_kv_fill_kernel<128><<<blocks, 256, 0, st>>>(prm);
    else jl::jl_kv_fill_kernel<64><<<blocks, 256, 0, st>>>(prm);
  } else {
    if (head_dim == 128) jl::jl_decode_append_kernel<128><<<blocks, 256, 0, st>>>(prm);
    else jl::jl_decode_append_kernel<64><<<blocks, 256, 0, st>>>(prm);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, fill ? "kv fill launch" : "decode append launch");
  return ok();
}

}  // namespace

// ===================================================================== ABI ==

extern "C" {

const char* jl_last_error(void) { return g_err.c_str(); }

int64_t jl_group_size(int64_t L, int64_t w_pretrained) {
  if (w_pretrained < 1 || L < 0) return -1;
  const int64_t g = (L + w_pretrained - 1) / w_pretrained;
  return g < 1 ? 1 : g;
}

int jl_decode_single_launch_enabled(void) { return JL_DECODE_LAST_CTA_MERGE ? 1 : 0; }

int jl_debug_bounds_enabled(void) {
#ifdef JL_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

jl_status jl_sync_status(jl_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, jl::g_status, sizeof word);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(jl::g_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    if (word & jl::kDevErrTimeout) return fail(JL_ERR_TIMEOUT, "a bounded in-kernel wait ran out");
    if (word & jl::kDevErrBounds)
      return fail(JL_ERR_INVALID, "a cache writer met a position outside the cache or the RoPE tables");
    if (word & jl::kDevErrIndex)
      return fail(JL_ERR_INVALID, "a debug-bounds check failed: a kernel derived an index outside its buffer");
  }
  return ok();
}

#ifdef JL_TRACE
// Copies the timeline of the traced CTA (a build with -DJL_TRACE only).
jl_status jl_debug_trace(long long* host, int n) {
  const cudaError_t e = cudaMemcpyFromSymbol(host, jl::g_trace, sizeof(long long) * (n < 4096 ? n : 4096));
  return e == cudaSuccess ? ok() : cuda_fail(e, "trace copy");
}
jl_status jl_debug_trace_decode(long long* host, int n) {
  const cudaError_t e = cudaMemcpyFromSymbol(host, jl::g_trace_dec, sizeof(long long) * (n < 1024 ? n : 1024));
  return e == cudaSuccess ? ok() : cuda_fail(e, "trace copy");
}
#endif

jl_status jl_selftest_wait_timeout(int64_t limit_cycles, jl_stream_t stream) {
  if (limit_cycles < 1000 || limit_cycles > 2000000000LL)
    return fail(JL_ERR_INVALID, "limit_cycles must be in [1000, 2e9] (got %lld)", (long long)limit_cycles);
  jl::jl_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ok();
}

jl_status jl_rope_tables_scaled(float* cos_out, float* sin_out, int64_t n_pos, int32_t head_dim, double rope_base,
                                const double* freq_scale, jl_stream_t stream) {
  if (!cos_out || !sin_out || !freq_scale) return fail(JL_ERR_INVALID, "null pointer argument");
  if (n_pos < 1) return fail(JL_ERR_INVALID, "n_pos must be >= 1 (got %lld)", (long long)n_pos);
  if (head_dim != 64 && head_dim != 128)
    return fail(JL_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (!(rope_base > 1.0)) return fail(JL_ERR_INVALID, "rope_base must be > 1");
  if (!aligned16(cos_out) || !aligned16(sin_out)) return fail(JL_ERR_INVALID, "tables must be 16-byte aligned");
  jl::FreqScale fs{};
  for (int c = 0; c < head_dim / 2; ++c) {
    if (!(freq_scale[c] > 0.0)) return fail(JL_ERR_INVALID, "freq_scale[%d] must be > 0", c);
    fs.lambda[c] = freq_scale[c];
  }
  const int half = head_dim / 2;
  const int64_t blocks64 = (n_pos * half + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(blocks64 < 148 * 64 ? blocks64 : 148 * 64);
  jl::jl_rope_table_scaled_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(cos_out, sin_out, n_pos,
                                                                                              half, rope_base, fs);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "scaled table launch");
  return ok();
}

jl_status jl_interp_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                            int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                            int32_t w0, const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                            const float* cos_rem, const float* sin_rem, int64_t n_rem_rows, float softmax_scale,
                            void* out, float* lse, void* workspace, size_t workspace_bytes, jl_stream_t stream) {
  if (!cos_rem || !sin_rem) return fail(JL_ERR_INVALID, "null remote table");
  if (n_rem_rows < max_seqlen)
    return fail(JL_ERR_INVALID, "n_rem_rows (%lld) must be >= max_seqlen (%d)", (long long)n_rem_rows, max_seqlen);
  if (!aligned16(cos_rem) || !aligned16(sin_rem)) return fail(JL_ERR_INVALID, "tables must be 16-byte aligned");
  jl::PrefillParams prm;
  bool empty;
  jl_status s = prefill_params(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, w0, 1, 0,
                               cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, &prm, &empty);
  if (s != JL_OK || empty) return s;
  prm.cos_rem = cos_rem;
  prm.sin_rem = sin_rem;
  prm.n_rem_rows = n_rem_rows;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (workspace == nullptr) return launch_prefill_any(q, k, v, prm, head_dim, st);
  // remote rows: the interpolated rotation at the raw position, for every sequence
  if ((s = rotate_keys(k, cu_seqlens, batch, total_tokens, Hkv, head_dim, 1, cos_tab, sin_tab, n_tab_rows, cos_rem,
                       sin_rem, n_rem_rows, workspace, workspace_bytes, st)) != JL_OK)
    return s;
  prm.krot = 1;
  return launch_prefill_any(q, workspace, v, prm, head_dim, st);
}

jl_status jl_rope_tables(float* cos_out, float* sin_out, int64_t n_pos, int32_t head_dim, double rope_base,
                         jl_stream_t stream) {
  if (!cos_out || !sin_out) return fail(JL_ERR_INVALID, "null table pointer");
  if (n_pos < 1) return fail(JL_ERR_INVALID, "n_pos must be >= 1 (got %lld)", (long long)n_pos);
  if (head_dim != 64 && head_dim != 128)
    return fail(JL_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  if (!(rope_base > 1.0)) return fail(JL_ERR_INVALID, "rope_base must be > 1");
  if (!aligned16(cos_out) || !aligned16(sin_out)) return fail(JL_ERR_INVALID, "tables must be 16-byte aligned");
  const int half = head_dim / 2;
  const int64_t total = n_pos * half;
  const int64_t blocks64 = (total + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(blocks64 < 148 * 64 ? blocks64 : 148 * 64);
  jl::jl_rope_table_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(cos_out, sin_out, n_pos,
                                                                                       half, rope_base);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  return ok();
}

jl_status jl_bifocal_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                             int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                             int32_t w0, int32_t w_pretrained, const float* cos_tab, const float* sin_tab,
                             int64_t n_tab_rows, float softmax_scale, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, jl_stream_t stream) {
  return prefill_common(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, w0, w_pretrained,
                        0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t jl_bifocal_prefill_workspace_size(int64_t total_tokens, int32_t Hkv, int32_t head_dim) {
  return key_rot_bytes(total_tokens, Hkv, head_dim);
}

jl_status jl_bifocal_prefill_and_cache(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                       int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t Hq,
                                       int32_t Hkv, int32_t head_dim, int32_t w0, int32_t w_pretrained,
                                       const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                                       float softmax_scale, void* out, float* lse, void* k_cache, void* v_cache,
                                       int64_t cache_stride, void* workspace, size_t workspace_bytes,
                                       jl_stream_t stream) {
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cache_stride < max_seqlen || cache_stride < 1)
    return fail(JL_ERR_INVALID, "cache_stride (%lld) must be >= max_seqlen (%d) and >= 1", (long long)cache_stride,
                max_seqlen);
  if (workspace != nullptr) {
    // Keys rotated once into the workspace: the attention is jl_bifocal_prefill's with
    // that workspace, and the cache writer fills the cache beside it.
    if (batch > 0 && total_tokens > 0 && max_seqlen > 0 && (!k_cache || !v_cache))
      return fail(JL_ERR_INVALID, "null cache pointer");
    jl_status s = prefill_common(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, w0,
                                 w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, workspace,
                                 workspace_bytes, st);
    if (s != JL_OK || batch == 0 || total_tokens == 0 || max_seqlen == 0) return s;
    return append_common(nullptr, k, v, cu_seqlens, nullptr, batch, total_tokens, 0, Hkv, head_dim, cos_tab,
                         sin_tab, n_tab_rows, nullptr, k_cache, v_cache, cache_stride, nullptr, 0, 0, 0, st, true);
  }
  jl::PrefillParams prm;
  bool empty;
  jl_status s = prefill_params(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, w0,
                               w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, &prm,
                               &empty);
  if (s != JL_OK || empty) return s;
  if (!k_cache || !v_cache) return fail(JL_ERR_INVALID, "null cache pointer");
  if (!aligned16(k_cache) || !aligned16(v_cache)) return fail(JL_ERR_INVALID, "caches must be 16-byte aligned");
  prm.k_cache_out = static_cast<__nv_bfloat16*>(k_cache);
  prm.v_cache_out = static_cast<__nv_bfloat16*>(v_cache);
  prm.v_raw = static_cast<const __nv_bfloat16*>(v);
  prm.cache_out_stride = cache_stride;
  if ((s = launch_prefill_any(q, k, v, prm, head_dim, st)) != JL_OK) return s;
  // With w0 = 0 and G > 1 no key tile is visited with base positions, so the kernel
  // cannot write R(j) k_j; the cache writer fills the cache instead.
  if (w0 == 0)
    return append_common(nullptr, k, v, cu_seqlens, nullptr, batch, total_tokens, 0, Hkv, head_dim, cos_tab,
                         sin_tab, n_tab_rows, nullptr, k_cache, v_cache, cache_stride, nullptr, 0, 0, 0, st, true);
  return ok();
}

jl_status jl_plain_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                           int64_t total_tokens, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                           const float* cos_tab, const float* sin_tab, int64_t n_tab_rows, float softmax_scale,
                           void* out, float* lse, void* workspace, size_t workspace_bytes, jl_stream_t stream) {
  return prefill_common(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, 0, 1, 1, cos_tab,
                        sin_tab, n_tab_rows, softmax_scale, out, lse, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

jl_status jl_kv_cache_fill(const void* k, const void* v, const int32_t* cu_seqlens, const int32_t* past_lens,
                           int32_t batch, int64_t total_tokens, int32_t Hkv, int32_t head_dim, const float* cos_tab,
                           const float* sin_tab, int64_t n_tab_rows, void* k_cache, void* v_cache,
                           int64_t cache_stride, jl_stream_t stream) {
  return append_common(nullptr, k, v, cu_seqlens, past_lens, batch, total_tokens, 0, Hkv, head_dim, cos_tab,
                       sin_tab, n_tab_rows, nullptr, k_cache, v_cache, cache_stride, nullptr, 0, 0, 0,
                       reinterpret_cast<cudaStream_t>(stream), true);
}

jl_status jl_kv_cache_fill_paged(const void* k, const void* v, const int32_t* cu_seqlens, const int32_t* past_lens,
                                 int32_t batch, int64_t total_tokens, int32_t Hkv, int32_t head_dim,
                                 const float* cos_tab, const float* sin_tab, int64_t n_tab_rows, void* k_pool,
                                 void* v_pool, const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                 int32_t num_pages, jl_stream_t stream) {
  if (page_size < 1 || max_pages < 1 || num_pages < 1)
    return fail(JL_ERR_INVALID, "page_size, max_pages and num_pages must be >= 1");
  if (batch > 0 && !block_table) return fail(JL_ERR_INVALID, "null block_table");
  return append_common(nullptr, k, v, cu_seqlens, past_lens, batch, total_tokens, 0, Hkv, head_dim, cos_tab,
                       sin_tab, n_tab_rows, nullptr, k_pool, v_pool, static_cast<int64_t>(max_pages) * page_size,
                       block_table, page_size, max_pages, num_pages, reinterpret_cast<cudaStream_t>(stream), true);
}

jl_status jl_decode_append_paged(const void* q, const void* k, const void* v, const int32_t* seqlens, int32_t B,
                                 int32_t Hq, int32_t Hkv, int32_t head_dim, const float* cos_tab,
                                 const float* sin_tab, int64_t n_tab_rows, void* q_out, void* k_pool, void* v_pool,
                                 const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                 int32_t num_pages, jl_stream_t stream) {
  if (page_size < 1 || max_pages < 1 || num_pages < 1)
    return fail(JL_ERR_INVALID, "page_size, max_pages and num_pages must be >= 1");
  if (B > 0 && !block_table) return fail(JL_ERR_INVALID, "null block_table");
  return append_common(q, k, v, seqlens, nullptr, B, 0, Hq, Hkv, head_dim, cos_tab, sin_tab, n_tab_rows, q_out,
                       k_pool, v_pool, static_cast<int64_t>(max_pages) * page_size, block_table, page_size,
                       max_pages, num_pages, reinterpret_cast<cudaStream_t>(stream), false);
}

jl_status jl_decode_append(const void* q, const void* k, const void* v, const int32_t* seqlens, int32_t B,
                           int32_t Hq, int32_t Hkv, int32_t head_dim, const float* cos_tab, const float* sin_tab,
                           int64_t n_tab_rows, void* q_out, void* k_cache, void* v_cache, int64_t cache_stride,
                           jl_stream_t stream) {
  return append_common(q, k, v, seqlens, nullptr, B, 0, Hq, Hkv, head_dim, cos_tab, sin_tab, n_tab_rows, q_out,
                       k_cache, v_cache, cache_stride, nullptr, 0, 0, 0, reinterpret_cast<cudaStream_t>(stream), false);
}

jl_status jl_bifocal_prefill_chunk(const void* q, const int32_t* cu_seqlens, const int32_t* past_lens, int32_t batch,
                                   int64_t total_tokens, int32_t max_seqlen, int32_t max_total, const void* k_cache,
                                   const void* v_cache, int64_t cache_stride, int32_t Hq, int32_t Hkv,
                                   int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                                   const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out,
                                   float* lse, jl_stream_t stream) {
  if (!past_lens && batch > 0) return fail(JL_ERR_INVALID, "past_lens is required");
  if (max_total < max_seqlen) return fail(JL_ERR_INVALID, "max_total must be >= max_seqlen");
  if (cache_stride < max_total)
    return fail(JL_ERR_INVALID, "cache_stride (%lld) must be >= max_total (%d)", (long long)cache_stride, max_total);
  if (static_cast<int64_t>(batch) * cache_stride > 0x7fffffffLL)
    return fail(JL_ERR_UNSUPPORTED, "batch * cache_stride must be < 2^31");
  if (n_tab_rows < max_total)
    return fail(JL_ERR_INVALID, "n_tab_rows (%lld) must be >= max_total (%d)", (long long)n_tab_rows, max_total);
  if (!aligned16(k_cache) || !aligned16(v_cache)) return fail(JL_ERR_INVALID, "caches must be 16-byte aligned");
  jl::PrefillParams prm;
  bool empty;
  jl_status s = prefill_params(q, k_cache, v_cache, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim,
                               w0, w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, &prm,
                               &empty);
  if (s != JL_OK || empty) return s;
  prm.cached = 1;
  prm.past_lens = past_lens;
  prm.cache_stride = cache_stride;
  return launch_prefill_any(q, k_cache, v_cache, prm, head_dim, reinterpret_cast<cudaStream_t>(stream));
}

size_t jl_bifocal_prefill_three_pass_workspace_size(int64_t total_tokens, int32_t Hq, int32_t head_dim) {
  return three_pass_ws_bytes(total_tokens, Hq, head_dim);
}

jl_status jl_bifocal_prefill_three_pass(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                        int32_t batch, int64_t total_tokens, int32_t max_seqlen, int32_t Hq,
                                        int32_t Hkv, int32_t head_dim, int32_t w0, int32_t w_pretrained,
                                        const float* cos_tab, const float* sin_tab, int64_t n_tab_rows,
                                        float softmax_scale, void* out, float* lse, void* workspace,
                                        size_t workspace_bytes, jl_stream_t stream) {
  jl::PrefillParams prm;
  bool empty;
  jl_status s = prefill_params(q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, Hq, Hkv, head_dim, w0,
                               w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, &prm, &empty);
  if (s != JL_OK || empty) return s;
  const size_t need = three_pass_ws_bytes(total_tokens, Hq, head_dim);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need)
    return fail(JL_ERR_INVALID, "three-pass workspace: %zu bytes needed, 16-byte aligned", need);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* o3x = static_cast<float*>(workspace);  // fp32: the merge subtracts pass 3 from pass 2
  const int64_t plane = total_tokens * Hq * head_dim;
  float* lse3x = reinterpret_cast<float*>(o3x + 3 * plane);
  const int modes[3] = {1, 0, 3};  // pass 1: window/base; pass 2: causal/remote (fused with w0 = 0); pass 3
  for (int pass = 0; pass < 3; ++pass) {
    jl::PrefillParams pp = prm;
    pp.mode = modes[pass];
    if (pass == 1) pp.w0 = 0;
    pp.out_f32 = o3x + pass * plane;
    pp.lse = lse3x + pass * total_tokens * Hq;
    if ((s = launch_prefill_any(q, k, v, pp, head_dim, st)) != JL_OK) return s;
  }
  const int64_t rows = total_tokens * Hq;
  const unsigned blocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  if (head_dim == 128)
    jl::jl_ie_merge_kernel<128><<<blocks, 256, 0, st>>>(o3x, lse3x, total_tokens, Hq, prm.out, lse);
  else
    jl::jl_ie_merge_kernel<64><<<blocks, 256, 0, st>>>(o3x, lse3x, total_tokens, Hq, prm.out, lse);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

jl_status jl_bifocal_decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                                  const int32_t* seqlens, int32_t B, int32_t max_pages, int32_t page_size,
                                  int32_t num_pages, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                                  int32_t w0, int32_t w_pretrained, const float* cos_tab, const float* sin_tab,
                                  int64_t n_tab_rows, float softmax_scale, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, jl_stream_t stream) {
  if (!decode_uses_tc(head_dim, Hq, Hkv < 1 ? 1 : Hkv) || Hkv < 1)
    return fail(JL_ERR_UNSUPPORTED, "paged decode needs head_dim 128 and Hq/Hkv <= 16");
  if (page_size < 128 || page_size % 128 != 0)
    return fail(JL_ERR_UNSUPPORTED, "page_size must be a positive multiple of 128 (got %d)", page_size);
  if (max_pages < 1 || static_cast<int64_t>(max_pages) * page_size < max_seqlen)
    return fail(JL_ERR_INVALID, "max_pages * page_size must cover max_seqlen");
  if (num_pages < 1 || static_cast<int64_t>(num_pages) * page_size > 0x7fffffffLL)
    return fail(JL_ERR_INVALID, "num_pages * page_size must be in [1, 2^31)");
  if (B > 0 && !block_table) return fail(JL_ERR_INVALID, "null block_table");
  // validated by the contiguous path with the pool as the cache rows, read through the block table
  return decode_common(q, k_pool, v_pool, seqlens, B, static_cast<int64_t>(num_pages) * page_size, max_seqlen, Hq,
                       Hkv, head_dim, w0, w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse,
                       workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), block_table, page_size,
                       max_pages);
}

size_t jl_bifocal_decode_workspace_size(int32_t B, int32_t Hq, int32_t head_dim, int32_t max_seqlen) {
  return decode_ws_bytes(B, Hq, head_dim, max_seqlen);
}

jl_status jl_bifocal_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                            int32_t B, int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv,
                            int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                            const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, jl_stream_t stream) {
  return decode_common(q, k_cache, v_cache, seqlens, B, cache_stride, max_seqlen, Hq, Hkv, head_dim, w0,
                       w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, workspace,
                       workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

jl_status jl_plain_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, int32_t B,
                          int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv, int32_t head_dim,
                          const float* cos_tab, const float* sin_tab, int64_t n_tab_rows, float softmax_scale,
                          void* out, float* lse, void* workspace, size_t workspace_bytes, jl_stream_t stream) {
  return decode_common(q, k_cache, v_cache, seqlens, B, cache_stride, max_seqlen, Hq, Hkv, head_dim, 0, 1, 1,
                       cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ======================================== decode without caller workspace ==
//
// For callers that cannot allocate device memory (see jl_bifocal_decode_noalloc
// in jetlong.h).  The split-K partials live in one file-scope device array that
// every GPU loading this library holds until the process exits.  Host code may
// not pass the array's name to a kernel (on the host it is only a stand-in), so
// the device address is looked up with cudaGetSymbolAddress while that device is
// current (see static_scratch_for).

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// The scratch of the device the call runs on.  The kernels go to the caller's
// stream, so that stream, the current device and the query buffer must all be on
// one device: the array's address is only valid there.  Outside stream capture
// the address is looked up again on every call (it changes if the device's
// context was reset and the module reloaded); inside a capture the address from
// the last uncaptured call on that device is used, so the first call on a device
// must not be captured.
jl_status static_scratch_for(cudaStream_t st, const void* q, void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(JL_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  int st_dev = -1;
  e = cudaStreamGetDevice(st, &st_dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamGetDevice");
  if (st_dev != dev)
    return fail(JL_ERR_INVALID, "jl_bifocal_decode_noalloc: the stream belongs to device %d but device %d is current",
                st_dev, dev);
  cudaPointerAttributes pa{};
  e = cudaPointerGetAttributes(&pa, q);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes(q)");
  if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged)
    return fail(JL_ERR_INVALID, "jl_bifocal_decode_noalloc: q is not device memory");
  if (pa.type == cudaMemoryTypeDevice && pa.device != dev)
    return fail(JL_ERR_INVALID, "jl_bifocal_decode_noalloc: q lives on device %d but device %d is current", pa.device,
                dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    g_scratch_addr[dev] = p;
  } else if (g_scratch_addr[dev] == nullptr) {
    return fail(JL_ERR_INVALID,
                "jl_bifocal_decode_noalloc: the first call on device %d must come before any stream capture", dev);
  }
  *addr = g_scratch_addr[dev];
  return JL_OK;
}

}  // namespace

extern "C" {

size_t jl_bifocal_decode_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

jl_status jl_bifocal_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                                    int32_t B, int64_t cache_stride, int32_t max_seqlen, int32_t Hq, int32_t Hkv,
                                    int32_t head_dim, int32_t w0, int32_t w_pretrained, const float* cos_tab,
                                    const float* sin_tab, int64_t n_tab_rows, float softmax_scale, void* out,
                                    float* lse, jl_stream_t stream) {
  const size_t need = decode_ws_bytes(B, Hq, head_dim, max_seqlen);
  if (need > kStaticScratchBytes)
    return fail(JL_ERR_INVALID,
                "jl_bifocal_decode_noalloc: B=%d, Hq=%d, head_dim=%d, max_seqlen=%d need %zu bytes of scratch, "
                "more than the %zu-byte static scratch; use jl_bifocal_decode with a caller workspace",
                B, Hq, head_dim, max_seqlen, need, kStaticScratchBytes);
  if (B <= 0) return decode_common(q, k_cache, v_cache, seqlens, B, cache_stride, max_seqlen, Hq, Hkv, head_dim,
                                   w0, w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse,
                                   nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
  if (!q) return fail(JL_ERR_INVALID, "null pointer argument");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  const jl_status s = static_scratch_for(st, q, &scratch);
  if (s != JL_OK) return s;
  // Every partial the merge reads is written earlier in the same call, and the merge
  // counters count a word with another call's tag as zero, so nothing in the scratch
  // needs clearing between calls.  If a split gives up (the device status word is
  // set), the merge writes NaN instead of blending stale partials.
  return decode_common(q, k_cache, v_cache, seqlens, B, cache_stride, max_seqlen, Hq, Hkv, head_dim, w0,
                       w_pretrained, 0, cos_tab, sin_tab, n_tab_rows, softmax_scale, out, lse, scratch,
                       kStaticScratchBytes, st);
}

}  // extern "C"
