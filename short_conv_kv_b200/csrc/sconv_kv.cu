// C ABI of the fused ShortConv K/V step: argument validation, launch
// geometry and kernel dispatch.  See include/sconv_kv.h for the contract.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "sconv_kv.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill.cuh"

namespace {

using sconv::StepParams;
using KernelFn = void (*)(StepParams);

thread_local char g_cuda_error[256] = "";

constexpr int kBlock = 256;  // threads per CTA (one 8-channel group each)
constexpr int kMaxTile = 32;
constexpr int kMinTile = 8;  // >= SCONV_KV_MAX_W - 1: tile 0 covers the halo

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int W, int D>
KernelFn prefill_fn() { return sconv::prefill_kernel<W, D>; }
template <int W, int D>
KernelFn decode_fn() { return sconv::decode_kernel<W, D>; }

template <int D>
KernelFn pick_w(bool decode, int W) {
  switch (W) {
    case 1: return decode ? decode_fn<1, D>() : prefill_fn<1, D>();
    case 2: return decode ? decode_fn<2, D>() : prefill_fn<2, D>();
    case 3: return decode ? decode_fn<3, D>() : prefill_fn<3, D>();
    case 4: return decode ? decode_fn<4, D>() : prefill_fn<4, D>();
    case 5: return decode ? decode_fn<5, D>() : prefill_fn<5, D>();
    case 6: return decode ? decode_fn<6, D>() : prefill_fn<6, D>();
    case 7: return decode ? decode_fn<7, D>() : prefill_fn<7, D>();
    case 8: return decode ? decode_fn<8, D>() : prefill_fn<8, D>();
    default: return nullptr;
  }
}

KernelFn pick(bool decode, int W, int D) {
  switch (D) {
    case 64: return pick_w<64>(decode, W);
    case 128: return pick_w<128>(decode, W);
    case 256: return pick_w<256>(decode, W);
    default: return nullptr;
  }
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

// Checks shared by both entry points; fills the common part of P.
int validate_common(const void* k, const void* v, int64_t row_stride,
                    const void* conv_w_k, const void* conv_w_v,
                    const float* gamma_k, const float* gamma_v, int W,
                    int num_kv_heads, int head_dim, void* conv_state,
                    int64_t state_pool_size, const int64_t* slot_mapping,
                    void* k_cache, void* v_cache,
                    const sconv_kv_cache_layout_t* layout, StepParams* P) {
  if (!k || !v || !conv_w_k || !conv_w_v || !gamma_k || !gamma_v ||
      !slot_mapping || !k_cache || !v_cache || !layout)
    return SCONV_KV_ERR_NULL;
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
  return SCONV_KV_OK;
}

int launch(KernelFn fn, dim3 grid, dim3 block, StepParams* P, void* stream) {
  void* args[] = {P};
  cudaError_t e = cudaLaunchKernel(reinterpret_cast<const void*>(fn), grid, block, args, 0,
                                   static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return SCONV_KV_ERR_CUDA;
  }
  g_cuda_error[0] = '\0';
  return SCONV_KV_OK;
}

// Threads per CTA: all channel groups when they fit, in whole warps.
dim3 block_for(int NG) {
  const int t = NG >= kBlock ? kBlock : ((NG + 31) / 32) * 32;
  return dim3(t);
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
  StepParams P;
  int rc = validate_common(k, v, row_stride, conv_w_k, conv_w_v, gamma_k, gamma_v, W,
                           num_kv_heads, head_dim, conv_state, state_pool_size,
                           slot_mapping, k_cache, v_cache, layout, &P);
  if (rc != SCONV_KV_OK) return rc;
  if (!cu_seqlens) return SCONV_KV_ERR_NULL;
  if (num_seqs < 0 || num_tokens < 0 || num_tokens > INT32_MAX) return SCONV_KV_ERR_SHAPE;
  if (num_seqs == 0 || num_tokens == 0) return SCONV_KV_OK;
  KernelFn fn = pick(false, W, head_dim);
  if (!fn) return SCONV_KV_ERR_UNSUPPORTED;

  P.num_tokens = num_tokens;
  P.cu_seqlens = cu_seqlens;
  P.num_seqs = num_seqs;
  P.eps = eps;
  P.state_indices = state_indices;
  P.err = err_flag;

  // Tile length: spread the tokens over one wave of resident CTAs when
  // there are few, cap the tile when there are many (more, shorter CTAs
  // balance better at the tail).  Tile >= W-1 keeps the old state inside
  // the first tile of each sequence.
  const dim3 block = block_for(P.NG);
  const int64_t ctas_y = (P.NG + block.x - 1) / block.x;
  const int64_t resident = static_cast<int64_t>(sm_count()) * (W <= 4 ? 2 : 1);
  int64_t tile = (num_tokens * ctas_y + resident - 1) / resident;
  if (tile > kMaxTile) tile = kMaxTile;
  if (tile < kMinTile) tile = kMinTile;
  P.tile = static_cast<int>(tile);
  const int64_t grid_x = num_tokens / tile + num_seqs;
  if (grid_x > INT32_MAX || ctas_y > 65535) return SCONV_KV_ERR_SHAPE;
  return launch(fn, dim3(static_cast<unsigned>(grid_x), static_cast<unsigned>(ctas_y)), block,
                &P, stream);
}

int sconv_kv_decode(const void* k, const void* v, int64_t row_stride, int batch,
                    const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
                    const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
                    void* conv_state, const int32_t* state_indices,
                    int64_t state_pool_size, const int64_t* slot_mapping, void* k_cache,
                    void* v_cache, const sconv_kv_cache_layout_t* layout, int* err_flag,
                    void* stream) {
  StepParams P;
  int rc = validate_common(k, v, row_stride, conv_w_k, conv_w_v, gamma_k, gamma_v, W,
                           num_kv_heads, head_dim, conv_state, state_pool_size,
                           slot_mapping, k_cache, v_cache, layout, &P);
  if (rc != SCONV_KV_OK) return rc;
  if (batch < 0) return SCONV_KV_ERR_SHAPE;
  if (batch == 0) return SCONV_KV_OK;
  KernelFn fn = pick(true, W, head_dim);
  if (!fn) return SCONV_KV_ERR_UNSUPPORTED;
  P.num_tokens = batch;
  P.num_seqs = batch;
  P.eps = eps;
  P.state_indices = state_indices;
  P.err = err_flag;
  const dim3 block = block_for(P.NG);
  const int64_t ctas_y = (P.NG + block.x - 1) / block.x;
  if (ctas_y > 65535) return SCONV_KV_ERR_SHAPE;
  return launch(fn, dim3(static_cast<unsigned>(batch), static_cast<unsigned>(ctas_y)), block,
                &P, stream);
}

}  // extern "C"
