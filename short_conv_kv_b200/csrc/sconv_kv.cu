// C ABI of the fused ShortConv K/V step: argument validation, launch
// geometry and kernel dispatch.  See include/sconv_kv.h for the contract.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "sconv_kv.h"
#include "common.cuh"
#include "instances.h"
#include "stages.cuh"

namespace {

using sconv::StepParams;

thread_local char g_cuda_error[256] = "";


bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using sconv::TmaFn;
using sconv::DecFn;

bool uses_layout_variants(const sconv_kv_options_t* opts) {
  return opts && (opts->gamma_head_stride != 0 || opts->state_positions != nullptr);
}
// Kernel instances live in their own translation units (compiled in
// parallel): bf16 or MXFP8 store, without or with the layout variants.
TmaFn pick_prefill(int W, int D, bool mx, bool lv) {
  if (mx) return lv ? sconv::pick_prefill_mx_lv(W, D) : sconv::pick_prefill_mx(W, D);
  return lv ? sconv::pick_prefill_bf16_lv(W, D) : sconv::pick_prefill_bf16(W, D);
}
DecFn pick_decode(int W, int D, bool mx, bool lv) { return sconv::pick_decode(W, D, mx, lv); }

// Host-side caches (SM counts, shared-memory attributes, scratch addresses)
// are shared by every host thread that calls the library.
std::mutex g_cache_mutex;

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  std::lock_guard<std::mutex> lock(g_cache_mutex);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

// Shared memory of one SM and the part of it each resident CTA reserves
// (cached per device).
void smem_per_sm(size_t* total, size_t* reserved_per_cta) {
  static size_t cached_total[64] = {0}, cached_res[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    *total = 228 * 1024;
    *reserved_per_cta = 1024;
    return;
  }
  std::lock_guard<std::mutex> lock(g_cache_mutex);
  if (!cached_total[dev]) {
    int t = 0, r = 0;
    if (cudaDeviceGetAttribute(&t, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        t <= 0)
      t = 228 * 1024;
    if (cudaDeviceGetAttribute(&r, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        r < 0)
      r = 1024;
    cudaGetLastError();
    cached_total[dev] = static_cast<size_t>(t);
    cached_res[dev] = static_cast<size_t>(r);
  }
  *total = cached_total[dev];
  *reserved_per_cta = cached_res[dev];
}

// CTAs of `fn` that fit on one SM with `threads` threads and `smem` bytes of
// dynamic shared memory (after the kernel has been opted into that size);
// `fallback` if the query fails.  Cached per device, kernel and size.
int resident_per_sm(const void* fn, int threads, size_t smem, int fallback) {
  static const void* c_fn[256];
  static int c_dev[256], c_threads[256], c_n[256];
  static size_t c_smem[256];
  static int n_cached = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return fallback;
  }
  {
    std::lock_guard<std::mutex> lock(g_cache_mutex);
    for (int i = 0; i < n_cached; ++i)
      if (c_fn[i] == fn && c_dev[i] == dev && c_threads[i] == threads && c_smem[i] == smem)
        return c_n[i];
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    return fallback;
  }
  std::lock_guard<std::mutex> lock(g_cache_mutex);
  if (n_cached < 256) {
    c_fn[n_cached] = fn;
    c_dev[n_cached] = dev;
    c_threads[n_cached] = threads;
    c_smem[n_cached] = smem;
    c_n[n_cached] = n;
    ++n_cached;
  }
  return n;
}

// Opt a kernel into `bytes` of dynamic shared memory (once per kernel and
// size; host-side attribute, not a stream operation).
bool smem_attr_set(const void* fn, size_t bytes) {
  static const void* done_fn[512];
  static int done_dev[512];
  static size_t done_bytes[512];
  static int n_done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(g_cache_mutex);
  // the attribute belongs to the function in one device's context
  for (int i = 0; i < n_done; ++i)
    if (done_fn[i] == fn && done_dev[i] == dev && done_bytes[i] >= bytes) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  for (int i = 0; i < n_done; ++i)
    if (done_fn[i] == fn && done_dev[i] == dev) {
      done_bytes[i] = bytes;
      return true;
    }
  if (n_done < 512) {
    done_fn[n_done] = fn;
    done_dev[n_done] = dev;
    done_bytes[n_done] = bytes;
    ++n_done;
  }
  return true;
}

// Checks shared by both entry points; fills the common part of P.
int validate_common(const void* k, const void* v, int64_t row_stride,
                    const void* conv_w_k, const void* conv_w_v,
                    const float* gamma_k, const float* gamma_v, int W,
                    int num_kv_heads, int head_dim, void* conv_state,
                    int64_t state_pool_size, const int64_t* slot_mapping,
                    void* k_cache, void* v_cache,
                    const sconv_kv_cache_layout_t* layout, StepParams* P,
                    uint8_t* k_scale = nullptr, uint8_t* v_scale = nullptr, bool mx = false) {
  if (!k || !v || !conv_w_k || !conv_w_v || !gamma_k || !gamma_v ||
      !slot_mapping || !k_cache || !v_cache || !layout)
    return SCONV_KV_ERR_NULL;
  if (mx && (!k_scale || !v_scale)) return SCONV_KV_ERR_NULL;
  if (W > 1 && !conv_state) return SCONV_KV_ERR_NULL;
  if (W < 1 || W > SCONV_KV_MAX_W) return SCONV_KV_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return SCONV_KV_ERR_SHAPE;
  if (num_kv_heads < 1 || num_kv_heads > (1 << 16)) return SCONV_KV_ERR_SHAPE;
  const int64_t C = static_cast<int64_t>(num_kv_heads) * head_dim;
  if (row_stride < C) return SCONV_KV_ERR_SHAPE;
  if (state_pool_size < 0) return SCONV_KV_ERR_SHAPE;
  if (layout->num_kv_heads != num_kv_heads || layout->head_dim != head_dim)
    return SCONV_KV_ERR_SHAPE;
  if (layout->num_pages < 0 || layout->page_size < 1) return SCONV_KV_ERR_SHAPE;
  if (layout->stride_head < head_dim || layout->stride_slot < 1 || layout->stride_page < 1)
    return SCONV_KV_ERR_SHAPE;
  if (row_stride % 8 != 0) return SCONV_KV_ERR_ALIGN;
  if (!aligned16(k) || !aligned16(v) || !aligned16(conv_w_k) || !aligned16(conv_w_v) ||
      !aligned16(gamma_k) || !aligned16(gamma_v) || !aligned16(k_cache) ||
      !aligned16(v_cache) || (conv_state && !aligned16(conv_state)))
    return SCONV_KV_ERR_ALIGN;
  if (layout->stride_head % 8 || layout->stride_slot % 8 || layout->stride_page % 8)
    return SCONV_KV_ERR_ALIGN;
  // MXFP8: a scale byte per 32 elements, so element strides are multiples of 32
  if (mx && (layout->stride_head % 32 || layout->stride_slot % 32 || layout->stride_page % 32))
    return SCONV_KV_ERR_ALIGN;

  memset(P, 0, sizeof(*P));
  P->k = static_cast<const uint16_t*>(k);
  P->v = static_cast<const uint16_t*>(v);
  P->row_stride = row_stride;
  P->w_k = static_cast<const uint16_t*>(conv_w_k);
  P->w_v = static_cast<const uint16_t*>(conv_w_v);
  P->gamma_k = gamma_k;
  P->gamma_v = gamma_v;
  P->inv_d = 1.0f / static_cast<float>(head_dim);
  P->C = static_cast<int>(C);
  P->NG = static_cast<int>(2 * C / 8);
  P->state = static_cast<uint16_t*>(conv_state);
  P->pool = state_pool_size;
  P->slots = slot_mapping;
  P->k_cache = static_cast<uint16_t*>(k_cache);
  P->v_cache = static_cast<uint16_t*>(v_cache);
  P->num_slots = layout->num_pages * layout->page_size;
  P->page_size = layout->page_size;
  P->stride_page = layout->stride_page;
  P->stride_slot = layout->stride_slot;
  P->stride_head = layout->stride_head;
  P->slot_linear = layout->stride_page == layout->page_size * layout->stride_slot;
  if (mx) {
    P->k_data = static_cast<uint8_t*>(k_cache);
    P->v_data = static_cast<uint8_t*>(v_cache);
    P->k_scale = k_scale;
    P->v_scale = v_scale;
    P->k_cache = nullptr;
    P->v_cache = nullptr;
  }
  return SCONV_KV_OK;
}

// Layout variants (per-head gamma stride, ring-buffer state positions).
int apply_options(const sconv_kv_options_t* opts, int head_dim, StepParams* P) {
  P->gamma_hs = 0;
  P->state_pos = nullptr;
  if (!opts) return SCONV_KV_OK;
  if (opts->gamma_head_stride != 0 && opts->gamma_head_stride != head_dim)
    return SCONV_KV_ERR_SHAPE;
  P->gamma_hs = opts->gamma_head_stride;
  P->state_pos = opts->state_positions;
  return SCONV_KV_OK;
}

// Launch with programmatic stream serialisation: the kernel may start
// while the previous kernel in the stream drains; it waits for that kernel
// (griddepcontrol.wait) before touching global memory.
int launch(const void* fn, dim3 grid, dim3 block, void** args, size_t smem, void* stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return SCONV_KV_ERR_CUDA;
  }
  g_cuda_error[0] = '\0';
  return SCONV_KV_OK;
}


int prefill_impl(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream, bool mx,
    uint8_t* k_scale, uint8_t* v_scale, const sconv_kv_options_t* opts) {
  // an empty call enqueues nothing; its pointers are not examined (empty
  // tensors may have NULL data pointers)
  if (num_seqs < 0 || num_tokens < 0 || num_tokens > INT32_MAX) return SCONV_KV_ERR_SHAPE;
  if (num_seqs == 0 || num_tokens == 0) return SCONV_KV_OK;
  StepParams P;
  int rc = validate_common(k, v, row_stride, conv_w_k, conv_w_v, gamma_k, gamma_v, W,
                           num_kv_heads, head_dim, conv_state, state_pool_size,
                           slot_mapping, k_cache, v_cache, layout, &P, k_scale, v_scale, mx);
  if (rc != SCONV_KV_OK) return rc;
  rc = apply_options(opts, head_dim, &P);
  if (rc != SCONV_KV_OK) return rc;
  if (!cu_seqlens) return SCONV_KV_ERR_NULL;
  TmaFn fn = pick_prefill(W, head_dim, mx, uses_layout_variants(opts));
  if (!fn) return SCONV_KV_ERR_UNSUPPORTED;
  // the kernel keeps cache row offsets in 32 bits, in units of 8 elements
  {
    const __int128 last_row =
        static_cast<__int128>(layout->num_pages > 0 ? layout->num_pages - 1 : 0) *
            layout->stride_page +
        static_cast<__int128>(layout->page_size - 1) * layout->stride_slot;
    if (last_row / 8 >= static_cast<__int128>(sconv::kNoRow)) return SCONV_KV_ERR_SHAPE;
  }

  P.num_tokens = num_tokens;
  P.cu_seqlens = cu_seqlens;
  P.num_seqs = num_seqs;
  P.eps = eps;
  P.state_indices = state_indices;
  P.err = err_flag;

  // Geometry: channel slices of <= 256 groups (y), one thread per group
  // (thread 0 also issues the copies); two CTAs per SM with a ~96 KB ring
  // each (W <= 4) or one with ~192 KB; as many persistent CTAs per slice as
  // are resident (x), each streaming a contiguous token range of at least
  // one stage.
  sconv::TmaGeom G;
  const int nt = sconv::prefill_threads(W, mx);  // threads (channel groups) per CTA
  G.slice = P.NG < nt ? P.NG : nt;
  const int ctas_y = (P.NG + G.slice - 1) / G.slice;
  const int stage_bytes = sconv::prefill_stage_bytes(W, mx);  // laid out for a full slice
  const int per_sm = sconv::prefill_ctas_per_sm(W, mx);
  // the ring: 192 KB of an SM's shared memory split among its CTAs
  int stages = (2 * sconv::kTmaRingBytes2 / per_sm) / stage_bytes;
  G.stages = stages < 2 ? 2 : (stages > 16 ? 16 : stages);
  // + per-warp slot-offset tables + per-thread gammas
  G.smem_ring = G.stages * stage_bytes + sconv::kTmaOffTableBytes +
                sconv::prefill_gamma_bytes(W, mx);
  // cu_seqlens is staged in shared memory only while per_sm CTAs still fit
  // on an SM with it (beyond that the CTAs read it from global memory):
  // staging must never cost a resident CTA
  const size_t smem_base = static_cast<size_t>(G.smem_ring) + 16 * G.stages + 48;
  const size_t cu_bytes = 4 * (static_cast<size_t>(num_seqs) + 1);
  size_t sm_total = 0, sm_reserved = 0;
  smem_per_sm(&sm_total, &sm_reserved);
  G.cu_smem = (num_seqs < sconv::kTmaCuSmemMax &&
               per_sm * (smem_base + cu_bytes + sm_reserved) <= sm_total) ? 1 : 0;
  G.timeout_ns = (opts && opts->wait_timeout_ns > 0)
                     ? static_cast<unsigned long long>(opts->wait_timeout_ns)
                     : 1000000000ull;
  G.withhold_first = (opts && opts->withhold_first_copy) ? 1 : 0;
  G.state_wait_only = (opts && opts->state_only_dependency) ? 1 : 0;
  const size_t smem = smem_base + (G.cu_smem ? cu_bytes : 0);
  if (!smem_attr_set(reinterpret_cast<const void*>(fn), smem)) {
    snprintf(g_cuda_error, sizeof g_cuda_error, "cudaFuncSetAttribute failed");
    return SCONV_KV_ERR_CUDA;
  }
  const dim3 block(((G.slice + 31) / 32) * 32);
  // persistent CTAs: as many as are resident at this shared-memory size
  // (never more, or the rest would run as a second wave)
  const int occ = resident_per_sm(reinterpret_cast<const void*>(fn), static_cast<int>(block.x),
                                  smem, per_sm);
  const int64_t resident = static_cast<int64_t>(sm_count()) * (occ < per_sm ? occ : per_sm);
  int64_t ctas = resident / ctas_y;
  const int R = sconv::prefill_rows(W);
  const int64_t by_tokens = (num_tokens + R - 1) / R;
  if (ctas > by_tokens) ctas = by_tokens;
  if (ctas < 1) ctas = 1;
  G.ctas = static_cast<int>(ctas);
  // a short bf16 launch (few chunks per CTA) takes the instance made for
  // its compute-bound tail, when it is resident on the same terms
  if (!mx && !uses_layout_variants(opts) &&
      num_tokens <= static_cast<int64_t>(G.ctas) * R * SCONV_PREFILL_SHORT_CHUNKS) {
    const TmaFn fs = sconv::pick_prefill_bf16_short(W, head_dim);
    if (fs && smem_attr_set(reinterpret_cast<const void*>(fs), smem) &&
        resident_per_sm(reinterpret_cast<const void*>(fs), static_cast<int>(block.x), smem,
                        per_sm) >= occ)
      fn = fs;
  }
#ifndef SCONV_PREFILL_SEQ_COST
#define SCONV_PREFILL_SEQ_COST 16  // tokens a sequence start is worth when cutting ranges
#endif
  G.seq_cost = SCONV_PREFILL_SEQ_COST;
  G.cut_q = static_cast<int>(num_tokens / ctas);
  G.cut_r = static_cast<int>(num_tokens % ctas);
  void* args[] = {&P, &G};
  return launch(reinterpret_cast<const void*>(fn), dim3(G.ctas, ctas_y), block, args, smem,
                stream);
}

int decode_impl(const void* k, const void* v, int64_t row_stride, int batch,
                const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
                const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
                void* conv_state, const int32_t* state_indices, int64_t state_pool_size,
                const int64_t* slot_mapping, void* k_cache, void* v_cache,
                const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream, bool mx,
                uint8_t* k_scale, uint8_t* v_scale, const sconv_kv_options_t* opts) {
  if (batch < 0) return SCONV_KV_ERR_SHAPE;
  if (batch == 0) return SCONV_KV_OK;  // nothing enqueued, pointers not examined
  StepParams P;
  int rc = validate_common(k, v, row_stride, conv_w_k, conv_w_v, gamma_k, gamma_v, W,
                           num_kv_heads, head_dim, conv_state, state_pool_size,
                           slot_mapping, k_cache, v_cache, layout, &P, k_scale, v_scale, mx);
  if (rc != SCONV_KV_OK) return rc;
  rc = apply_options(opts, head_dim, &P);
  if (rc != SCONV_KV_OK) return rc;
  DecFn fn = pick_decode(W, head_dim, mx, uses_layout_variants(opts));
  if (!fn) return SCONV_KV_ERR_UNSUPPORTED;
  P.num_tokens = batch;
  P.num_seqs = batch;
  P.eps = eps;
  P.state_indices = state_indices;
  P.err = err_flag;

  // Geometry: channel slices of <= 256 groups (y), one thread per group;
  // four CTAs per SM (fewer for W > 4) sharing ~192 KB of ring
  // (one stage = one sequence's W rows); enough CTAs (x) that each handles
  // at most kDecMaxSeqs sequences, and at least one resident wave.
  sconv::DecGeom G;
  G.slice = P.NG < 256 ? P.NG : 256;
  const int ctas_y = (P.NG + G.slice - 1) / G.slice;
  const int stage_bytes = W * G.slice * 16;
  const int per_sm = sconv::decode_ctas_per_sm(W);
  int stages = (192 * 1024 / per_sm) / stage_bytes;
  G.stages = stages < 2 ? 2 : (stages > 8 ? 8 : stages);
  G.smem_ring = G.stages * stage_bytes;
  G.timeout_ns = (opts && opts->wait_timeout_ns > 0)
                     ? static_cast<unsigned long long>(opts->wait_timeout_ns)
                     : 1000000000ull;
  G.withhold_first = (opts && opts->withhold_first_copy) ? 1 : 0;
  G.state_early = (opts && opts->independent_state) ? 1 : 0;
  int64_t ctas = static_cast<int64_t>(sm_count()) * per_sm / ctas_y;
  const int64_t need = (static_cast<int64_t>(batch) + sconv::kDecMaxSeqs - 1) / sconv::kDecMaxSeqs;
  if (ctas < need) ctas = need;
  if (ctas > batch) ctas = batch;
  if (ctas < 1) ctas = 1;
  G.ctas = static_cast<int>(ctas);
  if (ctas_y > 65535) return SCONV_KV_ERR_SHAPE;
  const size_t smem = static_cast<size_t>(G.smem_ring) + 16 * G.stages +
                      2 * sconv::kDecMaxSeqs * sizeof(long long) +
                      sconv::kDecMaxSeqs * sizeof(int) + 16;
  if (!smem_attr_set(reinterpret_cast<const void*>(fn), smem)) {
    snprintf(g_cuda_error, sizeof g_cuda_error, "cudaFuncSetAttribute failed");
    return SCONV_KV_ERR_CUDA;
  }
  const dim3 block(((G.slice + 31) / 32) * 32);
  void* args[] = {&P, &G};
  return launch(reinterpret_cast<const void*>(fn), dim3(G.ctas, ctas_y), block, args, smem,
                stream);
}

// ---- unfused stages

using StageFn = void (*)(sconv::StageParams);

template <int W>
StageFn stage_conv_fn() { return sconv::stage_conv_kernel<W>; }
template <int W>
StageFn stage_state_fn() { return sconv::stage_state_kernel<W>; }

StageFn stage_conv_by_w(int W) {
  switch (W) {
    case 1: return stage_conv_fn<1>();
    case 2: return stage_conv_fn<2>();
    case 3: return stage_conv_fn<3>();
    case 4: return stage_conv_fn<4>();
    case 5: return stage_conv_fn<5>();
    case 6: return stage_conv_fn<6>();
    case 7: return stage_conv_fn<7>();
    case 8: return stage_conv_fn<8>();
    default: return nullptr;
  }
}
StageFn stage_state_by_w(int W) {
  switch (W) {
    case 2: return stage_state_fn<2>();
    case 3: return stage_state_fn<3>();
    case 4: return stage_state_fn<4>();
    case 5: return stage_state_fn<5>();
    case 6: return stage_state_fn<6>();
    case 7: return stage_state_fn<7>();
    case 8: return stage_state_fn<8>();
    default: return nullptr;
  }
}
StageFn stage_rmsnorm_by_d(int D) {
  switch (D) {
    case 64: return sconv::stage_rmsnorm_kernel<64>;
    case 128: return sconv::stage_rmsnorm_kernel<128>;
    case 256: return sconv::stage_rmsnorm_kernel<256>;
    default: return nullptr;
  }
}

// Shape checks shared by the stages; fills the channel counts of P.
int stage_shape(int num_kv_heads, int head_dim, int64_t num_tokens, sconv::StageParams* P) {
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return SCONV_KV_ERR_SHAPE;
  if (num_kv_heads < 1 || num_kv_heads > (1 << 16)) return SCONV_KV_ERR_SHAPE;
  if (num_tokens < 0 || num_tokens > INT32_MAX) return SCONV_KV_ERR_SHAPE;
  memset(P, 0, sizeof(*P));
  P->C = num_kv_heads * head_dim;
  P->D = head_dim;
  P->NG = 2 * P->C / 8;
  P->num_tokens = num_tokens;
  P->inv_d = 1.0f / static_cast<float>(head_dim);
  return SCONV_KV_OK;
}

// Grid-stride launch over `work` items of one thread each.
int stage_launch(StageFn fn, int64_t work, sconv::StageParams* P, void* stream) {
  if (work <= 0) return SCONV_KV_OK;
  const int64_t want = (work + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  void* args[] = {P};
  return launch(reinterpret_cast<const void*>(fn), dim3(static_cast<unsigned>(want < cap ? want : cap)),
                dim3(256), args, 0, stream);
}

// ---- static scratch of the no-alloc unfused step (y, then z)

__device__ __align__(256) unsigned char g_noalloc_scratch[SCONV_KV_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch in the current device's context, looked up
// on every call (a host-side table lookup, no allocation): a cached address
// could outlive its context (cudaDeviceReset, or a caller that switches
// driver contexts).  nullptr if the lookup fails.
unsigned char* noalloc_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<unsigned char*>(p);
}

// ---- unfused stages: argument checks (nothing enqueued) and launches

int prep_stage_conv(const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
                    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
                    const void* conv_w_v, int W, int num_kv_heads, int head_dim,
                    const void* conv_state, const int32_t* state_indices,
                    int64_t state_pool_size, void* y, int* err_flag, sconv::StageParams* P) {
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, P);
  if (st) return st;
  if (!k || !v || !cu_seqlens || !conv_w_k || !conv_w_v || !y || (W > 1 && !conv_state))
    return SCONV_KV_ERR_NULL;
  if (W < 1 || W > SCONV_KV_MAX_W || num_seqs < 0 || state_pool_size < 0 || row_stride < P->C)
    return SCONV_KV_ERR_SHAPE;
  if (row_stride % 8 || !aligned16(k) || !aligned16(v) || !aligned16(conv_w_k) ||
      !aligned16(conv_w_v) || !aligned16(y) || (conv_state && !aligned16(conv_state)))
    return SCONV_KV_ERR_ALIGN;
  P->k = static_cast<const uint16_t*>(k);
  P->v = static_cast<const uint16_t*>(v);
  P->row_stride = row_stride;
  P->cu_seqlens = cu_seqlens;
  P->num_seqs = num_seqs;
  P->w_k = static_cast<const uint16_t*>(conv_w_k);
  P->w_v = static_cast<const uint16_t*>(conv_w_v);
  P->W = W;
  P->state = const_cast<uint16_t*>(static_cast<const uint16_t*>(conv_state));
  P->state_indices = state_indices;
  P->pool = state_pool_size;
  P->y = static_cast<uint16_t*>(y);
  P->err = err_flag;
  return SCONV_KV_OK;
}

int prep_stage_rmsnorm(const void* y, int64_t num_tokens, const float* gamma_k,
                       const float* gamma_v, float eps, int num_kv_heads, int head_dim, void* z,
                       sconv::StageParams* P) {
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, P);
  if (st) return st;
  if (!y || !gamma_k || !gamma_v || !z) return SCONV_KV_ERR_NULL;
  if (!aligned16(y) || !aligned16(z) || !aligned16(gamma_k) || !aligned16(gamma_v))
    return SCONV_KV_ERR_ALIGN;
  P->y = const_cast<uint16_t*>(static_cast<const uint16_t*>(y));
  P->z = static_cast<uint16_t*>(z);
  P->gamma_k = gamma_k;
  P->gamma_v = gamma_v;
  P->eps = eps;
  return SCONV_KV_OK;
}

int prep_stage_scatter(const void* z, int64_t num_tokens, int num_kv_heads, int head_dim,
                       const int64_t* slot_mapping, void* k_cache, void* v_cache,
                       const sconv_kv_cache_layout_t* layout, const int32_t* cu_seqlens,
                       int num_seqs, int W, const int32_t* state_indices,
                       int64_t state_pool_size, int* err_flag, sconv::StageParams* P) {
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, P);
  if (st) return st;
  if (!z || !slot_mapping || !k_cache || !v_cache || !layout) return SCONV_KV_ERR_NULL;
  if (cu_seqlens && (num_seqs < 1 || W < 1 || W > SCONV_KV_MAX_W || state_pool_size < 0))
    return SCONV_KV_ERR_SHAPE;
  if (layout->num_kv_heads != num_kv_heads || layout->head_dim != head_dim ||
      layout->num_pages < 0 || layout->page_size < 1 || layout->stride_head < head_dim ||
      layout->stride_slot < 1 || layout->stride_page < 1)
    return SCONV_KV_ERR_SHAPE;
  if (!aligned16(z) || !aligned16(k_cache) || !aligned16(v_cache) || layout->stride_head % 8 ||
      layout->stride_slot % 8 || layout->stride_page % 8)
    return SCONV_KV_ERR_ALIGN;
  P->z = const_cast<uint16_t*>(static_cast<const uint16_t*>(z));
  P->slots = slot_mapping;
  P->k_cache = static_cast<uint16_t*>(k_cache);
  P->v_cache = static_cast<uint16_t*>(v_cache);
  P->num_slots = layout->num_pages * layout->page_size;
  P->page_size = layout->page_size;
  P->stride_page = layout->stride_page;
  P->stride_slot = layout->stride_slot;
  P->stride_head = layout->stride_head;
  P->cu_seqlens = cu_seqlens;
  P->num_seqs = cu_seqlens ? num_seqs : 0;
  P->W = cu_seqlens ? W : 1;
  P->state_indices = state_indices;
  P->pool = state_pool_size;
  P->err = err_flag;
  return SCONV_KV_OK;
}

int prep_stage_state(const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
                     const int32_t* cu_seqlens, int num_seqs, int W, int num_kv_heads,
                     int head_dim, void* conv_state, const int32_t* state_indices,
                     int64_t state_pool_size, int* err_flag, sconv::StageParams* P) {
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, P);
  if (st) return st;
  if (W < 1 || W > SCONV_KV_MAX_W || num_seqs < 0 || state_pool_size < 0 || row_stride < P->C)
    return SCONV_KV_ERR_SHAPE;
  if (W == 1 || num_seqs == 0) return SCONV_KV_OK;  // no state rows: nothing to launch
  if (!k || !v || !cu_seqlens || !conv_state) return SCONV_KV_ERR_NULL;
  if (row_stride % 8 || !aligned16(k) || !aligned16(v) || !aligned16(conv_state))
    return SCONV_KV_ERR_ALIGN;
  P->k = static_cast<const uint16_t*>(k);
  P->v = static_cast<const uint16_t*>(v);
  P->row_stride = row_stride;
  P->cu_seqlens = cu_seqlens;
  P->num_seqs = num_seqs;
  P->W = W;
  P->state = static_cast<uint16_t*>(conv_state);
  P->state_indices = state_indices;
  P->pool = state_pool_size;
  P->err = err_flag;
  return SCONV_KV_OK;
}

int launch_stage_conv(sconv::StageParams* P, void* stream) {
  return stage_launch(stage_conv_by_w(P->W), P->num_tokens * P->NG, P, stream);
}
int launch_stage_rmsnorm(sconv::StageParams* P, void* stream) {
  return stage_launch(stage_rmsnorm_by_d(P->D), P->num_tokens * P->NG, P, stream);
}
int launch_stage_scatter(sconv::StageParams* P, void* stream) {
  return stage_launch(sconv::stage_scatter_kernel, P->num_tokens * P->NG, P, stream);
}
int launch_stage_state(sconv::StageParams* P, void* stream) {
  if (P->W <= 1 || P->num_seqs == 0) return SCONV_KV_OK;
  return stage_launch(stage_state_by_w(P->W), static_cast<int64_t>(P->num_seqs) * P->NG, P,
                      stream);
}

}  // namespace

extern "C" {

int sconv_kv_version(void) { return 100; }

const char* sconv_kv_strerror(int status) {
  switch (status) {
    case SCONV_KV_OK: return "ok";
    case SCONV_KV_ERR_NULL: return "a required pointer is NULL";
    case SCONV_KV_ERR_SHAPE: return "bad shape (W, head_dim, heads, counts, strides or layout)";
    case SCONV_KV_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case SCONV_KV_ERR_UNSUPPORTED: return "unsupported combination";
    case SCONV_KV_ERR_CUDA: return "CUDA error at launch (see sconv_kv_last_cuda_error)";
    case SCONV_KV_ERR_SCRATCH: return "call needs more than the static scratch buffer";
    default: return "unknown status";
  }
}

const char* sconv_kv_last_cuda_error(void) { return g_cuda_error; }

int sconv_kv_cache_layout(int64_t num_pages, int64_t page_size, int num_kv_heads,
                          int head_dim, sconv_kv_cache_layout_t* out) {
  if (!out) return SCONV_KV_ERR_NULL;
  if (num_pages < 0 || page_size < 1 || num_kv_heads < 1 || head_dim < 1)
    return SCONV_KV_ERR_SHAPE;
  out->num_pages = num_pages;
  out->page_size = page_size;
  out->num_kv_heads = num_kv_heads;
  out->head_dim = head_dim;
  out->stride_head = head_dim;
  out->stride_slot = static_cast<int64_t>(num_kv_heads) * head_dim;
  out->stride_page = page_size * out->stride_slot;
  out->bytes_per_cache = num_pages * out->stride_page * 2;
  return SCONV_KV_OK;
}

int sconv_kv_prefill_varlen(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream) {
  return prefill_impl(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
                      gamma_k, gamma_v, eps, W, num_kv_heads, head_dim, conv_state,
                      state_indices, state_pool_size, slot_mapping, k_cache, v_cache, layout,
                      err_flag, stream, false, nullptr, nullptr, nullptr);
}

int sconv_kv_decode(const void* k, const void* v, int64_t row_stride, int batch,
                    const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
                    const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
                    void* conv_state, const int32_t* state_indices,
                    int64_t state_pool_size, const int64_t* slot_mapping, void* k_cache,
                    void* v_cache, const sconv_kv_cache_layout_t* layout, int* err_flag,
                    void* stream) {
  return decode_impl(k, v, row_stride, batch, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, W,
                     num_kv_heads, head_dim, conv_state, state_indices, state_pool_size,
                     slot_mapping, k_cache, v_cache, layout, err_flag, stream, false, nullptr,
                     nullptr, nullptr);
}

int sconv_kv_prefill_varlen_mxfp8(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_data, uint8_t* k_scale, void* v_data,
    uint8_t* v_scale, const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream) {
  return prefill_impl(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
                      gamma_k, gamma_v, eps, W, num_kv_heads, head_dim, conv_state,
                      state_indices, state_pool_size, slot_mapping, k_data, v_data, layout,
                      err_flag, stream, true, k_scale, v_scale, nullptr);
}

int sconv_kv_decode_mxfp8(const void* k, const void* v, int64_t row_stride, int batch,
                          const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
                          const float* gamma_v, float eps, int W, int num_kv_heads,
                          int head_dim, void* conv_state, const int32_t* state_indices,
                          int64_t state_pool_size, const int64_t* slot_mapping, void* k_data,
                          uint8_t* k_scale, void* v_data, uint8_t* v_scale,
                          const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream) {
  return decode_impl(k, v, row_stride, batch, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, W,
                     num_kv_heads, head_dim, conv_state, state_indices, state_pool_size,
                     slot_mapping, k_data, v_data, layout, err_flag, stream, true, k_scale,
                     v_scale, nullptr);
}

int sconv_kv_prefill_varlen_ex(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, const sconv_kv_options_t* options,
    int* err_flag, void* stream) {
  return prefill_impl(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
                      gamma_k, gamma_v, eps, W, num_kv_heads, head_dim, conv_state,
                      state_indices, state_pool_size, slot_mapping, k_cache, v_cache, layout,
                      err_flag, stream, false, nullptr, nullptr, options);
}

int sconv_kv_decode_ex(const void* k, const void* v, int64_t row_stride, int batch,
                       const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
                       const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
                       void* conv_state, const int32_t* state_indices,
                       int64_t state_pool_size, const int64_t* slot_mapping, void* k_cache,
                       void* v_cache, const sconv_kv_cache_layout_t* layout,
                       const sconv_kv_options_t* options, int* err_flag, void* stream) {
  return decode_impl(k, v, row_stride, batch, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, W,
                     num_kv_heads, head_dim, conv_state, state_indices, state_pool_size,
                     slot_mapping, k_cache, v_cache, layout, err_flag, stream, false, nullptr,
                     nullptr, options);
}

int sconv_kv_prefill_varlen_mxfp8_ex(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_data, uint8_t* k_scale, void* v_data,
    uint8_t* v_scale, const sconv_kv_cache_layout_t* layout,
    const sconv_kv_options_t* options, int* err_flag, void* stream) {
  return prefill_impl(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
                      gamma_k, gamma_v, eps, W, num_kv_heads, head_dim, conv_state,
                      state_indices, state_pool_size, slot_mapping, k_data, v_data, layout,
                      err_flag, stream, true, k_scale, v_scale, options);
}

int sconv_kv_decode_mxfp8_ex(const void* k, const void* v, int64_t row_stride, int batch,
                             const void* conv_w_k, const void* conv_w_v,
                             const float* gamma_k, const float* gamma_v, float eps, int W,
                             int num_kv_heads, int head_dim, void* conv_state,
                             const int32_t* state_indices, int64_t state_pool_size,
                             const int64_t* slot_mapping, void* k_data, uint8_t* k_scale,
                             void* v_data, uint8_t* v_scale,
                             const sconv_kv_cache_layout_t* layout,
                             const sconv_kv_options_t* options, int* err_flag, void* stream) {
  return decode_impl(k, v, row_stride, batch, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, W,
                     num_kv_heads, head_dim, conv_state, state_indices, state_pool_size,
                     slot_mapping, k_data, v_data, layout, err_flag, stream, true, k_scale,
                     v_scale, options);
}

int sconv_kv_unfused_step_noalloc(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream) {
  // shape limits first, so the scratch size below cannot overflow
  sconv::StageParams shape;
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, &shape);
  if (st) return st;
  if (num_seqs < 0) return SCONV_KV_ERR_SHAPE;
  if (num_tokens == 0 || num_seqs == 0) return SCONV_KV_OK;
  // num_tokens < 2^31, channels <= 2^24: the product stays below 2^58
  const int64_t bytes = num_tokens * 2 * static_cast<int64_t>(num_kv_heads) * head_dim * 2;
  const int64_t part = (bytes + 255) / 256 * 256;
  if (2 * part > SCONV_KV_NOALLOC_SCRATCH_BYTES) return SCONV_KV_ERR_SCRATCH;
  unsigned char* scratch = noalloc_scratch();
  if (!scratch) {
    snprintf(g_cuda_error, sizeof g_cuda_error, "scratch address lookup failed");
    return SCONV_KV_ERR_CUDA;
  }
  void* y = scratch;
  void* z = scratch + part;
  // every stage's arguments are checked before the first launch, so an
  // argument error leaves nothing enqueued
  sconv::StageParams Pc, Pn, Ps, Pu;
  st = prep_stage_conv(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
                       W, num_kv_heads, head_dim, conv_state, state_indices, state_pool_size, y,
                       err_flag, &Pc);
  if (st) return st;
  st = prep_stage_rmsnorm(y, num_tokens, gamma_k, gamma_v, eps, num_kv_heads, head_dim, z, &Pn);
  if (st) return st;
  st = prep_stage_scatter(z, num_tokens, num_kv_heads, head_dim, slot_mapping, k_cache, v_cache,
                          layout, cu_seqlens, num_seqs, W, state_indices, state_pool_size,
                          err_flag, &Ps);
  if (st) return st;
  st = prep_stage_state(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, W, num_kv_heads,
                        head_dim, conv_state, state_indices, state_pool_size, err_flag, &Pu);
  if (st) return st;
  if ((st = launch_stage_conv(&Pc, stream))) return st;
  if ((st = launch_stage_rmsnorm(&Pn, stream))) return st;
  if ((st = launch_stage_scatter(&Ps, stream))) return st;
  return launch_stage_state(&Pu, stream);
}

int sconv_kv_stage_conv(const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
                        const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
                        const void* conv_w_v, int W, int num_kv_heads, int head_dim,
                        const void* conv_state, const int32_t* state_indices,
                        int64_t state_pool_size, void* y, int* err_flag, void* stream) {
  sconv::StageParams P;
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, &P);
  if (st) return st;
  if (num_tokens == 0 || num_seqs == 0) return SCONV_KV_OK;
  st = prep_stage_conv(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
                       W, num_kv_heads, head_dim, conv_state, state_indices, state_pool_size, y,
                       err_flag, &P);
  if (st) return st;
  return launch_stage_conv(&P, stream);
}

int sconv_kv_stage_rmsnorm(const void* y, int64_t num_tokens, const float* gamma_k,
                           const float* gamma_v, float eps, int num_kv_heads, int head_dim,
                           void* z, void* stream) {
  sconv::StageParams P;
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, &P);
  if (st) return st;
  if (num_tokens == 0) return SCONV_KV_OK;
  st = prep_stage_rmsnorm(y, num_tokens, gamma_k, gamma_v, eps, num_kv_heads, head_dim, z, &P);
  if (st) return st;
  return launch_stage_rmsnorm(&P, stream);
}

int sconv_kv_stage_scatter(const void* z, int64_t num_tokens, int num_kv_heads, int head_dim,
                           const int64_t* slot_mapping, void* k_cache, void* v_cache,
                           const sconv_kv_cache_layout_t* layout, const int32_t* cu_seqlens,
                           int num_seqs, int W, const int32_t* state_indices,
                           int64_t state_pool_size, int* err_flag, void* stream) {
  sconv::StageParams P;
  int st = stage_shape(num_kv_heads, head_dim, num_tokens, &P);
  if (st) return st;
  if (num_tokens == 0) return SCONV_KV_OK;
  st = prep_stage_scatter(z, num_tokens, num_kv_heads, head_dim, slot_mapping, k_cache, v_cache,
                          layout, cu_seqlens, num_seqs, W, state_indices, state_pool_size,
                          err_flag, &P);
  if (st) return st;
  return launch_stage_scatter(&P, stream);
}

int sconv_kv_stage_state_update(const void* k, const void* v, int64_t row_stride,
                                int64_t num_tokens, const int32_t* cu_seqlens, int num_seqs,
                                int W, int num_kv_heads, int head_dim, void* conv_state,
                                const int32_t* state_indices, int64_t state_pool_size,
                                int* err_flag, void* stream) {
  sconv::StageParams P;
  int st = prep_stage_state(k, v, row_stride, num_tokens, cu_seqlens, num_seqs, W, num_kv_heads,
                            head_dim, conv_state, state_indices, state_pool_size, err_flag, &P);
  if (st) return st;
  return launch_stage_state(&P, stream);
}

}  // extern "C"
