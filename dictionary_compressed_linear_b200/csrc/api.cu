// C ABI of libdictproj: validation, handles, uploads and forward dispatch.
// Every entry point validates its arguments before touching the device and
// reports failures through a status code plus a thread-local message.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dictproj.h"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {

static thread_local char g_err[512] = "";

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return status;
}
void clear_error() { g_err[0] = 0; }

int cuda_fail(cudaError_t e, const char* what) {
  return fail(DICTPROJ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Host-side fault injection for error-path tests: DICTPROJ_FAULT=alloc|copy.
static bool fault(const char* kind) {
  const char* f = std::getenv("DICTPROJ_FAULT");
  return f && std::strcmp(f, kind) == 0;
}

static cudaError_t dmalloc(void** p, size_t n) {
  if (fault("alloc")) return cudaErrorMemoryAllocation;
  return cudaMalloc(p, n ? n : 16);
}
static cudaError_t h2d(void* d, const void* h, size_t n) {
  if (fault("copy")) return cudaErrorInvalidValue;
  return n ? cudaMemcpy(d, h, n, cudaMemcpyHostToDevice) : cudaSuccess;
}

// One-time per-device set-up (kernel attributes) and capability check.
static std::atomic<int> g_decode_kernels{DICTPROJ_DECODE_AUTO};

// Whether a decode call goes to the fused kernel: FUSED always tries it; SPLIT
// and AUTO never while the two-kernel path is the faster one on every LLaMA-7B
// shape measured on B200 (chained calls, M = 1: 7.9 vs 13.8 us for 4096x2048x4096,
// 13.3 vs 25.6 us for 4096x3072x11008, 12.5 vs 23.2 us for 11008x3072x4096); AUTO
// still takes the fused kernel for calls the two-kernel path cannot serve
// (non-NVFP4 coefficient values, or a Z table beyond its shared memory).
static bool use_fused(int n, const dictproj_group* const* g, const dictproj_layer* const* l, const __half* const* x,
                      int M, int dev, FusedLaunchPlan* fp) {
  const int which = g_decode_kernels.load(std::memory_order_relaxed);
  if (which == DICTPROJ_DECODE_SPLIT) return false;
  if (which == DICTPROJ_DECODE_AUTO) {
    bool split_ok = coeff_smem_fits(g[0]->k, decode_mp(M), dev);
    for (int i = 0; i < n; ++i) split_ok = split_ok && l[i]->cfmt == DICTPROJ_CFMT_NVFP4 && coeff_smem_fits(g[i]->k, decode_mp(M), dev);
    if (split_ok) return false;
  }
  return fused_plan_launch(n, g, l, x, M, smem_optin_of(dev), fp);
}

static std::mutex g_dev_mu;
static std::vector<int> g_dev_ready;

int ensure_device(int* dev_out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if ((int)g_dev_ready.size() <= dev) g_dev_ready.resize(dev + 1, 0);
  if (!g_dev_ready[dev]) {
    cudaDeviceProp prop;
    if ((e = cudaGetDeviceProperties(&prop, dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10)
      return fail(DICTPROJ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                  prop.major, prop.minor);
    if ((e = prepare_decode_kernels(dev)) != cudaSuccess) return cuda_fail(e, "kernel set-up");
    if ((e = prepare_prefill_kernels(dev)) != cudaSuccess) return cuda_fail(e, "prefill kernel set-up");
    if ((e = prepare_fused_kernels(dev)) != cudaSuccess) return cuda_fail(e, "fused kernel set-up");
    if ((e = prepare_index_kernels(dev)) != cudaSuccess) return cuda_fail(e, "index-format kernel set-up");
    g_dev_ready[dev] = 1;
  }
  *dev_out = dev;
  return DICTPROJ_OK;
}

static int check_group_shape(int d_in, int k) {
  if (d_in <= 0 || k <= 0 || d_in % 32 || k % 16)
    return fail(DICTPROJ_ERR_SHAPE, "group: need d_in > 0 with d_in %% 32 == 0 and k > 0 with k %% 16 == 0 (got d_in=%d k=%d)", d_in, k);
  if (k > 65535) return fail(DICTPROJ_ERR_SHAPE, "group: k=%d exceeds 65535", k);
  return DICTPROJ_OK;
}

}  // namespace dictproj

using namespace dictproj;

extern "C" {

const char* dictproj_last_error(void) { return g_err; }

const char* dictproj_status_string(int s) {
  switch (s) {
    case DICTPROJ_OK: return "DICTPROJ_OK";
    case DICTPROJ_ERR_NULL: return "DICTPROJ_ERR_NULL";
    case DICTPROJ_ERR_SHAPE: return "DICTPROJ_ERR_SHAPE";
    case DICTPROJ_ERR_ALIGN: return "DICTPROJ_ERR_ALIGN";
    case DICTPROJ_ERR_MISMATCH: return "DICTPROJ_ERR_MISMATCH";
    case DICTPROJ_ERR_RANGE: return "DICTPROJ_ERR_RANGE";
    case DICTPROJ_ERR_CUDA: return "DICTPROJ_ERR_CUDA";
    case DICTPROJ_ERR_OOM: return "DICTPROJ_ERR_OOM";
    case DICTPROJ_ERR_TIMEOUT: return "DICTPROJ_ERR_TIMEOUT";
    case DICTPROJ_ERR_UNSUPPORTED: return "DICTPROJ_ERR_UNSUPPORTED";
    case DICTPROJ_ERR_VALUE: return "DICTPROJ_ERR_VALUE";
    case DICTPROJ_ERR_IO: return "DICTPROJ_ERR_IO";
    default: return "DICTPROJ_ERR_UNKNOWN";
  }
}

int dictproj_version(void) { return 10000; }

int dictproj_group_packed_sizes(int d_in, int k, size_t* codes_bytes, size_t* scales_bytes) {
  clear_error();
  if (!codes_bytes || !scales_bytes) return fail(DICTPROJ_ERR_NULL, "group_packed_sizes: NULL output");
  if (d_in <= 0 || k <= 0 || d_in % 16) return fail(DICTPROJ_ERR_SHAPE, "group_packed_sizes: need d_in %% 16 == 0 and k > 0");
  *codes_bytes = (size_t)d_in * k / 2;
  *scales_bytes = (size_t)d_in * k / 16;
  return DICTPROJ_OK;
}

int dictproj_pack_group_host(const float* D, int d_in, int k, uint8_t* codes, uint8_t* scales, float* s_D) {
  clear_error();
  return pack_group_host(D, d_in, k, codes, scales, s_D);
}

int dictproj_layer_packed_entries(const int32_t* col_ptr, int k, int d_out, size_t* total) {
  clear_error();
  return layer_packed_entries(col_ptr, k, d_out, total);
}

int dictproj_pack_layer_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                             int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes,
                             uint8_t* scales, uint8_t* idx, uint16_t* seg_start, float* s_C) {
  clear_error();
  return pack_layer_host(col_ptr, atom_idx, vals, k, d_out, pcol_ptr, nnz, codes, scales, idx, seg_start, s_C);
}

int dictproj_pack_layer_blocks_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                                    int d_out, uint32_t* blk_ptr, uint16_t* blk_idx, uint8_t* codes, uint8_t* scales,
                                    float* s_C) {
  clear_error();
  return pack_layer_blocks_host(col_ptr, atom_idx, vals, k, d_out, blk_ptr, blk_idx, codes, scales, s_C);
}

int dictproj_pack_layer_bitmap_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                                    int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes, uint8_t* scales,
                                    uint32_t* bitmap, float* s_C) {
  clear_error();
  return pack_layer_bitmap_host(col_ptr, atom_idx, vals, k, d_out, pcol_ptr, nnz, codes, scales, bitmap, s_C);
}

int dictproj_cfmt_value_bytes(int fmt) {
  switch (fmt) {
    case DICTPROJ_CFMT_FP16: return 2;
    case DICTPROJ_CFMT_FP8:
    case DICTPROJ_CFMT_INT8: return 1;
    default: return 0;
  }
}

int dictproj_pack_layer_fmt_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                                 int d_out, int fmt, uint32_t* pcol_ptr, uint32_t* nnz, void* values,
                                 uint8_t* idx, uint16_t* seg_start, float* s_C) {
  clear_error();
  return pack_layer_fmt_host(col_ptr, atom_idx, vals, k, d_out, fmt, pcol_ptr, nnz, values, idx, seg_start, s_C);
}

void dictproj_free_group(dictproj_group* g) {
  if (!g) return;
  cudaFree(g->codes);
  cudaFree(g->scales);
  cudaFree(g->z32);
  cudaFree(g->z16);
  cudaFree(g->cdense);
  cudaFree(g->fcodes);
  cudaFree(g->fscales);
  cudaFree(g->zx);
  cudaFree(g->fsync);
  delete g;
}

void dictproj_free_layer(dictproj_layer* l) {
  if (!l) return;
  cudaFree(l->col_ptr);
  cudaFree(l->codes);
  cudaFree(l->scales);
  cudaFree(l->idx);
  cudaFree(l->seg_start);
  cudaFree(l->cplan_off);
  cudaFree(l->cplan);
  cudaFree(l->bitmap);
  cudaFree(l->blk_ptr);
  cudaFree(l->blk_idx);
  delete l;
}

int dictproj_group_upload(const uint8_t* codes, const uint8_t* scales, float s_D, int d_in, int k,
                          int max_tokens, dictproj_group** out) {
  clear_error();
  if (!codes || !scales || !out) return fail(DICTPROJ_ERR_NULL, "group_upload: NULL pointer");
  *out = nullptr;
  int st = check_group_shape(d_in, k);
  if (st) return st;
  if (max_tokens < 1) return fail(DICTPROJ_ERR_RANGE, "group_upload: max_tokens must be >= 1 (got %d)", max_tokens);
  if (!(s_D > 0.0f) || !std::isfinite(s_D)) return fail(DICTPROJ_ERR_VALUE, "group_upload: s_D must be finite and > 0");
  int dev;
  if ((st = ensure_device(&dev))) return st;
  dictproj_group* g = new (std::nothrow) dictproj_group();
  if (!g) return fail(DICTPROJ_ERR_OOM, "group_upload: host allocation failed");
  g->device = dev;
  g->d_in = d_in;
  g->k = k;
  g->max_tokens = max_tokens;
  g->s = s_D;
  g->codes_bytes = (size_t)d_in * k / 2;
  g->scales_bytes = (size_t)d_in * k / 16;
  cudaError_t e;
  if ((e = cudaDeviceGetAttribute(&g->n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) {
    delete g;
    return cuda_fail(e, "group_upload: SM count");
  }
  g->zslices = dict_max_slices(d_in, k, g->n_sm);
  const size_t zbytes = (size_t)g->zslices * k * kDecodeMaxTokens * sizeof(float);
  const size_t z16bytes = (size_t)max_tokens * k * sizeof(uint16_t);
  if ((e = dmalloc((void**)&g->codes, g->codes_bytes)) || (e = dmalloc((void**)&g->scales, g->scales_bytes)) ||
      (e = dmalloc((void**)&g->z32, zbytes)) || (e = dmalloc((void**)&g->z16, z16bytes))) {
    dictproj_free_group(g);
    cudaGetLastError();
    return fail(DICTPROJ_ERR_OOM, "group_upload: device allocation failed (%s)", cudaGetErrorName(e));
  }
  if ((e = h2d(g->codes, codes, g->codes_bytes)) || (e = h2d(g->scales, scales, g->scales_bytes)) ||
      (e = cudaMemset(g->z32, 0, zbytes))) {
    dictproj_free_group(g);
    cudaGetLastError();
    return cuda_fail(e, "group_upload: copy to device");
  }
  if ((e = encode_dict_codes_map(g, &g->codes_map)) != cudaSuccess) {
    dictproj_free_group(g);
    return cuda_fail(e, "group_upload: tensor map of the dictionary codes");
  }
  bool fused = false;
  if (fault("alloc") || (e = fused_group_setup(g, codes, scales, &fused)) != cudaSuccess) {
    dictproj_free_group(g);
    cudaGetLastError();
    return fail(DICTPROJ_ERR_OOM, "group_upload: fused decode buffers (%s)", cudaGetErrorName(e));
  }
  *out = g;
  return DICTPROJ_OK;
}

int dictproj_pack_group(const float* D, int d_in, int k, int max_tokens, dictproj_group** out) {
  clear_error();
  if (!D || !out) return fail(DICTPROJ_ERR_NULL, "pack_group: NULL pointer");
  *out = nullptr;
  int st = check_group_shape(d_in, k);
  if (st) return st;
  if (max_tokens < 1) return fail(DICTPROJ_ERR_RANGE, "pack_group: max_tokens must be >= 1 (got %d)", max_tokens);
  std::vector<uint8_t> codes, scales;
  try {
    codes.resize((size_t)d_in * k / 2);
    scales.resize((size_t)d_in * k / 16);
  } catch (...) {
    return fail(DICTPROJ_ERR_OOM, "pack_group: host allocation failed");
  }
  float s = 0.f;
  if ((st = pack_group_host(D, d_in, k, codes.data(), scales.data(), &s))) return st;
  return dictproj_group_upload(codes.data(), scales.data(), s, d_in, k, max_tokens, out);
}

int dictproj_group_reserve_prefill(dictproj_group* g, int max_d_out) {
  clear_error();
  if (!g) return fail(DICTPROJ_ERR_NULL, "group_reserve_prefill: NULL handle");
  if (max_d_out < 1) return fail(DICTPROJ_ERR_RANGE, "group_reserve_prefill: max_d_out=%d < 1", max_d_out);
  if (max_d_out <= g->cdense_cols) return DICTPROJ_OK;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "group_reserve_prefill: cudaGetDevice");
  if (dev != g->device)
    return fail(DICTPROJ_ERR_MISMATCH, "group_reserve_prefill: current device %d, group on device %d", dev, g->device);
  uint16_t* p = nullptr;
  if ((e = dmalloc((void**)&p, (size_t)max_d_out * g->k * sizeof(uint16_t))) != cudaSuccess) {
    cudaGetLastError();
    return fail(DICTPROJ_ERR_OOM, "group_reserve_prefill: device allocation failed (%s)", cudaGetErrorName(e));
  }
  // the old buffer may still be read by queued work of this group
  if (g->cdense && (e = cudaDeviceSynchronize()) != cudaSuccess) {
    cudaFree(p);
    return cuda_fail(e, "group_reserve_prefill: synchronise before freeing the old scratch");
  }
  cudaFree(g->cdense);
  g->cdense = p;
  g->cdense_cols = max_d_out;
  return DICTPROJ_OK;
}

// Upload of a packed C_l in format fmt: NVFP4 (codes + scales) or FP16 / FP8 /
// INT8 (values in `codes`, one per stored entry; `scales` unused).
static int layer_upload_impl(const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                             const uint8_t* idx, const uint16_t* seg_start, float s_C, int k, int d_out, int fmt,
                             dictproj_layer** out) {
  if (!pcol_ptr || !codes || (fmt == DICTPROJ_CFMT_NVFP4 && !scales) || !idx || !seg_start || !out)
    return fail(DICTPROJ_ERR_NULL, "layer_upload: NULL pointer");
  if (fmt < DICTPROJ_CFMT_NVFP4 || fmt > DICTPROJ_CFMT_INT8)
    return fail(DICTPROJ_ERR_RANGE, "layer_upload: unknown coefficient format %d", fmt);
  *out = nullptr;
  if (k <= 0 || k % 16 || k > 65535 || d_out <= 0)
    return fail(DICTPROJ_ERR_SHAPE, "layer_upload: need 0 < k <= 65535, k %% 16 == 0, d_out > 0 (got k=%d d_out=%d)", k, d_out);
  if (!(s_C > 0.0f) || !std::isfinite(s_C)) return fail(DICTPROJ_ERR_VALUE, "layer_upload: s_C must be finite and > 0");
  if (pcol_ptr[0] != 0) return fail(DICTPROJ_ERR_RANGE, "layer_upload: col_ptr[0] must be 0");
  const int nseg = (k + 255) / 256;
  for (int o = 0; o < d_out; ++o) {
    const uint32_t n = pcol_ptr[o + 1] - pcol_ptr[o];
    if (pcol_ptr[o + 1] < pcol_ptr[o] || n % 16 || n > (uint32_t)((k + 15) / 16 * 16))
      return fail(DICTPROJ_ERR_RANGE, "layer_upload: column %d has a bad padded length %u", o, n);
    const uint16_t* ss = seg_start + (size_t)o * nseg;
    if (ss[0] != 0) return fail(DICTPROJ_ERR_RANGE, "layer_upload: seg_start[%d][0] != 0", o);
    for (int s = 1; s < nseg; ++s)
      if (ss[s] < ss[s - 1] || ss[s] > n) return fail(DICTPROJ_ERR_RANGE, "layer_upload: seg_start of column %d not monotone", o);
    // every entry's atom 256*s(q) + idx[q] must be < k (the kernels index Z with it)
    int s = 0;
    for (uint32_t q = 0; q < n; ++q) {
      while (s + 1 < nseg && ss[s + 1] <= q) ++s;
      if (256 * s + (int)idx[pcol_ptr[o] + q] >= k)
        return fail(DICTPROJ_ERR_RANGE, "layer_upload: column %d entry %u addresses atom >= k", o, q);
    }
  }
  int dev, st;
  if ((st = ensure_device(&dev))) return st;
  dictproj_layer* l = new (std::nothrow) dictproj_layer();
  if (!l) return fail(DICTPROJ_ERR_OOM, "layer_upload: host allocation failed");
  l->device = dev;
  l->k = k;
  l->d_out = d_out;
  l->nseg = nseg;
  l->s = s_C;
  l->total = pcol_ptr[d_out];
  l->cfmt = fmt;
  const size_t T = l->total;
  const size_t code_bytes = fmt == DICTPROJ_CFMT_NVFP4 ? T / 2 : T * (size_t)dictproj_cfmt_value_bytes(fmt);
  const size_t scale_bytes = fmt == DICTPROJ_CFMT_NVFP4 ? T / 16 : 0;
  cudaError_t e;
  // +16 bytes on every array so rounded-up copy ranges stay inside the allocation
  if ((e = dmalloc((void**)&l->col_ptr, (d_out + 1) * sizeof(uint32_t) + 16)) ||
      (e = dmalloc((void**)&l->codes, code_bytes + 16)) || (e = dmalloc((void**)&l->scales, scale_bytes + 16)) ||
      (e = dmalloc((void**)&l->idx, T + 16)) ||
      (e = dmalloc((void**)&l->seg_start, (size_t)d_out * nseg * sizeof(uint16_t) + 16))) {
    dictproj_free_layer(l);
    cudaGetLastError();
    return fail(DICTPROJ_ERR_OOM, "layer_upload: device allocation failed (%s)", cudaGetErrorName(e));
  }
  if ((e = h2d(l->col_ptr, pcol_ptr, (d_out + 1) * sizeof(uint32_t))) || (e = h2d(l->codes, codes, code_bytes)) ||
      (e = h2d(l->scales, scales, scale_bytes)) || (e = h2d(l->idx, idx, T)) ||
      (e = h2d(l->seg_start, seg_start, (size_t)d_out * nseg * sizeof(uint16_t)))) {
    dictproj_free_layer(l);
    cudaGetLastError();
    return cuda_fail(e, "layer_upload: copy to device");
  }
  int n_sm = 0;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) {
    dictproj_free_layer(l);
    return cuda_fail(e, "layer_upload: device attributes");
  }
  l->n_sm = n_sm;
  l->gather_ok = fmt == DICTPROJ_CFMT_NVFP4 && gather_supported(pcol_ptr, d_out, nseg);
  {  // column chunks of the fused decode kernel
    std::vector<uint32_t> off;
    std::vector<uint4> chunks;
    int maxc = 0;
    l->fused_ok = fused_layer_plan(pcol_ptr, d_out, nseg, fmt, n_sm, off, chunks, &maxc);
    l->cplan_max = maxc;
    if (l->fused_ok) {
      if ((e = dmalloc((void**)&l->cplan_off, off.size() * sizeof(uint32_t))) ||
          (e = dmalloc((void**)&l->cplan, std::max<size_t>(1, chunks.size()) * sizeof(uint4)))) {
        dictproj_free_layer(l);
        cudaGetLastError();
        return fail(DICTPROJ_ERR_OOM, "layer_upload: device allocation failed (%s)", cudaGetErrorName(e));
      }
      if ((e = h2d(l->cplan_off, off.data(), off.size() * sizeof(uint32_t))) ||
          (e = h2d(l->cplan, chunks.data(), chunks.size() * sizeof(uint4)))) {
        dictproj_free_layer(l);
        cudaGetLastError();
        return cuda_fail(e, "layer_upload: copy to device");
      }
    }
  }
  // the true entry count is not part of the packed arrays; dictproj_pack_layer records it
  l->nnz_total = 0;
  *out = l;
  return DICTPROJ_OK;
}

int dictproj_layer_upload(const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                          const uint8_t* idx, const uint16_t* seg_start, float s_C, int k, int d_out,
                          dictproj_layer** out) {
  clear_error();
  return layer_upload_impl(pcol_ptr, codes, scales, idx, seg_start, s_C, k, d_out, DICTPROJ_CFMT_NVFP4, out);
}

int dictproj_layer_upload_fmt(const uint32_t* pcol_ptr, const void* values, const uint8_t* idx,
                              const uint16_t* seg_start, float s_C, int k, int d_out, int fmt,
                              dictproj_layer** out) {
  clear_error();
  if (fmt == DICTPROJ_CFMT_NVFP4)
    return fail(DICTPROJ_ERR_RANGE, "layer_upload_fmt: NVFP4 layers are uploaded by dictproj_layer_upload");
  return layer_upload_impl(pcol_ptr, static_cast<const uint8_t*>(values), nullptr, idx, seg_start, s_C, k, d_out, fmt,
                           out);
}

int dictproj_pack_layer_fmt(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                            int fmt, dictproj_layer** out) {
  clear_error();
  if (!col_ptr || !out) return fail(DICTPROJ_ERR_NULL, "pack_layer_fmt: NULL pointer");
  *out = nullptr;
  if (fmt == DICTPROJ_CFMT_NVFP4) return dictproj_pack_layer(col_ptr, atom_idx, vals, k, d_out, out);
  if (k <= 0 || k % 16) return fail(DICTPROJ_ERR_SHAPE, "pack_layer_fmt: k must be a positive multiple of 16 (got %d)", k);
  if (fmt < DICTPROJ_CFMT_FP16 || fmt > DICTPROJ_CFMT_INT8)
    return fail(DICTPROJ_ERR_RANGE, "pack_layer_fmt: unknown coefficient format %d", fmt);
  size_t total = 0;
  int st = layer_packed_entries(col_ptr, k, d_out, &total);
  if (st) return st;
  const int nseg = (k + 255) / 256;
  std::vector<uint32_t> pptr, nnz;
  std::vector<uint8_t> values, idx;
  std::vector<uint16_t> ss;
  try {
    pptr.resize(d_out + 1);
    nnz.resize(d_out);
    values.resize(total * (size_t)dictproj_cfmt_value_bytes(fmt) + 2);
    idx.resize(total + 1);
    ss.resize((size_t)d_out * nseg);
  } catch (...) {
    return fail(DICTPROJ_ERR_OOM, "pack_layer_fmt: host allocation failed");
  }
  float s = 0.f;
  if ((st = pack_layer_fmt_host(col_ptr, atom_idx, vals, k, d_out, fmt, pptr.data(), nnz.data(), values.data(),
                                idx.data(), ss.data(), &s)))
    return st;
  if ((st = layer_upload_impl(pptr.data(), values.data(), nullptr, idx.data(), ss.data(), s, k, d_out, fmt, out)))
    return st;
  (*out)->nnz_total = (size_t)col_ptr[d_out];
  return DICTPROJ_OK;
}

int dictproj_layer_format(const dictproj_layer* l, int* fmt) {
  clear_error();
  if (!l || !fmt) return fail(DICTPROJ_ERR_NULL, "layer_format: NULL pointer");
  *fmt = l->cfmt;
  return DICTPROJ_OK;
}

int dictproj_layer_export_fmt(const dictproj_layer* l, uint32_t* pcol_ptr, void* values, uint8_t* idx,
                              uint16_t* seg_start, float* s_C) {
  clear_error();
  if (!l || !pcol_ptr || !values || !idx || !seg_start || !s_C)
    return fail(DICTPROJ_ERR_NULL, "layer_export_fmt: NULL pointer");
  if (l->cfmt == DICTPROJ_CFMT_NVFP4)
    return fail(DICTPROJ_ERR_UNSUPPORTED, "layer_export_fmt: an NVFP4 layer is exported by dictproj_layer_export");
  const size_t T = l->total;
  cudaError_t e;
  if ((e = cudaMemcpy(pcol_ptr, l->col_ptr, (l->d_out + 1) * sizeof(uint32_t), cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(values, l->codes, T * (size_t)dictproj_cfmt_value_bytes(l->cfmt), cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(idx, l->idx, T, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(seg_start, l->seg_start, (size_t)l->d_out * l->nseg * sizeof(uint16_t), cudaMemcpyDeviceToHost)))
    return cuda_fail(e, "layer_export_fmt");
  *s_C = l->s;
  return DICTPROJ_OK;
}

int dictproj_pack_layer(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                        dictproj_layer** out) {
  clear_error();
  if (!col_ptr || !out) return fail(DICTPROJ_ERR_NULL, "pack_layer: NULL pointer");
  *out = nullptr;
  if (k <= 0 || k % 16) return fail(DICTPROJ_ERR_SHAPE, "pack_layer: k must be a positive multiple of 16 (got %d)", k);
  size_t total = 0;
  int st = layer_packed_entries(col_ptr, k, d_out, &total);
  if (st) return st;
  const int nseg = (k + 255) / 256;
  std::vector<uint32_t> pptr, nnz;
  std::vector<uint8_t> codes, scales, idx;
  std::vector<uint16_t> ss;
  try {
    pptr.resize(d_out + 1);
    nnz.resize(d_out);
    codes.resize(total / 2 + 1);
    scales.resize(total / 16 + 1);
    idx.resize(total + 1);
    ss.resize((size_t)d_out * nseg);
  } catch (...) {
    return fail(DICTPROJ_ERR_OOM, "pack_layer: host allocation failed");
  }
  float s = 0.f;
  if ((st = pack_layer_host(col_ptr, atom_idx, vals, k, d_out, pptr.data(), nnz.data(), codes.data(),
                            scales.data(), idx.data(), ss.data(), &s)))
    return st;
  if ((st = dictproj_layer_upload(pptr.data(), codes.data(), scales.data(), idx.data(), ss.data(), s, k, d_out, out)))
    return st;
  (*out)->nnz_total = (size_t)col_ptr[d_out];
  return DICTPROJ_OK;
}

int dictproj_pack(const float* D, int d_in, int k, int max_tokens, int n_layers, const int32_t* const* col_ptr,
                  const int32_t* const* atom_idx, const float* const* vals, const int* d_out,
                  dictproj_group** group_out, dictproj_layer** layers_out) {
  clear_error();
  if (!group_out || !layers_out || (n_layers > 0 && (!col_ptr || !atom_idx || !vals || !d_out)))
    return fail(DICTPROJ_ERR_NULL, "pack: NULL pointer");
  if (n_layers < 0) return fail(DICTPROJ_ERR_SHAPE, "pack: n_layers < 0");
  *group_out = nullptr;
  for (int i = 0; i < n_layers; ++i) layers_out[i] = nullptr;
  int st = dictproj_pack_group(D, d_in, k, max_tokens, group_out);
  if (st) return st;
  for (int i = 0; i < n_layers; ++i) {
    if ((st = dictproj_pack_layer(col_ptr[i], atom_idx[i], vals[i], k, d_out[i], &layers_out[i]))) {
      for (int j = 0; j < i; ++j) {
        dictproj_free_layer(layers_out[j]);
        layers_out[j] = nullptr;
      }
      dictproj_free_group(*group_out);
      *group_out = nullptr;
      return st;
    }
  }
  if (max_tokens > kDecodeMaxTokens && n_layers > 0) {  // prefill scratch for these layers
    int dmax = 0;
    for (int i = 0; i < n_layers; ++i) dmax = d_out[i] > dmax ? d_out[i] : dmax;
    if ((st = dictproj_group_reserve_prefill(*group_out, dmax))) {
      for (int i = 0; i < n_layers; ++i) {
        dictproj_free_layer(layers_out[i]);
        layers_out[i] = nullptr;
      }
      dictproj_free_group(*group_out);
      *group_out = nullptr;
      return st;
    }
  }
  return DICTPROJ_OK;
}

int dictproj_group_export(const dictproj_group* g, uint8_t* codes, uint8_t* scales, float* s_D) {
  clear_error();
  if (!g || !codes || !scales || !s_D) return fail(DICTPROJ_ERR_NULL, "group_export: NULL pointer");
  cudaError_t e;
  if ((e = cudaMemcpy(codes, g->codes, g->codes_bytes, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(scales, g->scales, g->scales_bytes, cudaMemcpyDeviceToHost)))
    return cuda_fail(e, "group_export");
  *s_D = g->s;
  return DICTPROJ_OK;
}

int dictproj_layer_export(const dictproj_layer* l, uint32_t* pcol_ptr, uint8_t* codes, uint8_t* scales,
                          uint8_t* idx, uint16_t* seg_start, float* s_C) {
  clear_error();
  if (!l || !pcol_ptr || !codes || !scales || !idx || !seg_start || !s_C)
    return fail(DICTPROJ_ERR_NULL, "layer_export: NULL pointer");
  if (l->cfmt != DICTPROJ_CFMT_NVFP4)
    return fail(DICTPROJ_ERR_UNSUPPORTED, "layer_export: the layer's values are not NVFP4; use dictproj_layer_export_fmt");
  if (l->ifmt != DICTPROJ_IFMT_U8)
    return fail(DICTPROJ_ERR_UNSUPPORTED, "layer_export: the layer has a bitmap or block index; use "
                                          "dictproj_layer_export_bitmap / dictproj_layer_export_blocks");
  const size_t T = l->total;
  cudaError_t e;
  if ((e = cudaMemcpy(pcol_ptr, l->col_ptr, (l->d_out + 1) * sizeof(uint32_t), cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(codes, l->codes, T / 2, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(scales, l->scales, T / 16, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(idx, l->idx, T, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(seg_start, l->seg_start, (size_t)l->d_out * l->nseg * sizeof(uint16_t), cudaMemcpyDeviceToHost)))
    return cuda_fail(e, "layer_export");
  *s_C = l->s;
  return DICTPROJ_OK;
}

// ---- bitmap and block-structured C_l ---------------------------------------------------
// A layer struct with the common fields set and the index-format arrays empty.
static int new_index_layer(int k, int d_out, float s_C, int ifmt, dictproj_layer** out) {
  int dev, st;
  if ((st = ensure_device(&dev))) return st;
  dictproj_layer* l = new (std::nothrow) dictproj_layer();
  if (!l) return fail(DICTPROJ_ERR_OOM, "layer upload: host allocation failed");
  l->device = dev;
  l->k = k;
  l->d_out = d_out;
  l->nseg = (k + 255) / 256;
  l->s = s_C;
  l->cfmt = DICTPROJ_CFMT_NVFP4;
  l->ifmt = ifmt;
  l->gather_ok = false;  // the gather and fused kernels read the u8 index only
  l->fused_ok = false;
  cudaError_t e;
  int n_sm = 0;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) {
    delete l;
    return cuda_fail(e, "layer upload: device attributes");
  }
  l->n_sm = n_sm;
  *out = l;
  return DICTPROJ_OK;
}

int dictproj_layer_upload_bitmap(const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                                 const uint32_t* bitmap, float s_C, int k, int d_out, dictproj_layer** out) {
  clear_error();
  if (!pcol_ptr || !codes || !scales || !bitmap || !out) return fail(DICTPROJ_ERR_NULL, "layer_upload_bitmap: NULL pointer");
  *out = nullptr;
  if (k <= 0 || k % 16 || k > 65535 || d_out <= 0)
    return fail(DICTPROJ_ERR_SHAPE, "layer_upload_bitmap: need 0 < k <= 65535, k %% 16 == 0, d_out > 0 (got k=%d d_out=%d)", k, d_out);
  if (!(s_C > 0.0f) || !std::isfinite(s_C)) return fail(DICTPROJ_ERR_VALUE, "layer_upload_bitmap: s_C must be finite and > 0");
  if (pcol_ptr[0] != 0) return fail(DICTPROJ_ERR_RANGE, "layer_upload_bitmap: col_ptr[0] must be 0");
  const int words = (k + 31) / 32;
  size_t nnz = 0;
  for (int o = 0; o < d_out; ++o) {
    const uint32_t n = pcol_ptr[o + 1] - pcol_ptr[o];
    if (pcol_ptr[o + 1] < pcol_ptr[o] || n % 16 || n > (uint32_t)((k + 15) / 16 * 16))
      return fail(DICTPROJ_ERR_RANGE, "layer_upload_bitmap: column %d has a bad padded length %u", o, n);
    uint32_t bits = 0;
    for (int w = 0; w < words; ++w) {
      const uint32_t b = bitmap[(size_t)o * words + w];
      if (32 * w + 32 > k && (b >> (k - 32 * w)) != 0u && k - 32 * w < 32)
        return fail(DICTPROJ_ERR_RANGE, "layer_upload_bitmap: column %d marks atoms >= k", o);
      bits += (uint32_t)__builtin_popcount(b);
    }
    // the set bits are the stored entries; the padded length leaves less than one block of padding
    if (bits > n || n - bits >= 16)
      return fail(DICTPROJ_ERR_RANGE, "layer_upload_bitmap: column %d has %u retained atoms for %u stored entries", o,
                  bits, n);
    nnz += bits;
  }
  int st;
  dictproj_layer* l = nullptr;
  if ((st = new_index_layer(k, d_out, s_C, DICTPROJ_IFMT_BITMAP, &l))) return st;
  l->total = pcol_ptr[d_out];
  l->nnz_total = nnz;
  l->words = words;
  const size_t T = l->total;
  cudaError_t e;
  if ((e = dmalloc((void**)&l->col_ptr, (d_out + 1) * sizeof(uint32_t) + 16)) ||
      (e = dmalloc((void**)&l->codes, T / 2 + 16)) || (e = dmalloc((void**)&l->scales, T / 16 + 16)) ||
      (e = dmalloc((void**)&l->bitmap, (size_t)d_out * words * sizeof(uint32_t) + 16))) {
    dictproj_free_layer(l);
    cudaGetLastError();
    return fail(DICTPROJ_ERR_OOM, "layer_upload_bitmap: device allocation failed (%s)", cudaGetErrorName(e));
  }
  if ((e = h2d(l->col_ptr, pcol_ptr, (d_out + 1) * sizeof(uint32_t))) || (e = h2d(l->codes, codes, T / 2)) ||
      (e = h2d(l->scales, scales, T / 16)) ||
      (e = h2d(l->bitmap, bitmap, (size_t)d_out * words * sizeof(uint32_t)))) {
    dictproj_free_layer(l);
    cudaGetLastError();
    return cuda_fail(e, "layer_upload_bitmap: copy to device");
  }
  *out = l;
  return DICTPROJ_OK;
}

int dictproj_pack_layer_bitmap(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                               dictproj_layer** out) {
  clear_error();
  if (!col_ptr || !out) return fail(DICTPROJ_ERR_NULL, "pack_layer_bitmap: NULL pointer");
  *out = nullptr;
  size_t total = 0;
  int st = layer_packed_entries(col_ptr, k, d_out, &total);
  if (st) return st;
  const int words = (k + 31) / 32;
  std::vector<uint32_t> pptr, nnz, bitmap;
  std::vector<uint8_t> codes, scales;
  try {
    pptr.resize(d_out + 1);
    nnz.resize(d_out);
    bitmap.resize((size_t)d_out * words);
    codes.resize(total / 2 + 1);
    scales.resize(total / 16 + 1);
  } catch (...) {
    return fail(DICTPROJ_ERR_OOM, "pack_layer_bitmap: host allocation failed");
  }
  float s = 0.f;
  if ((st = pack_layer_bitmap_host(col_ptr, atom_idx, vals, k, d_out, pptr.data(), nnz.data(), codes.data(),
                                   scales.data(), bitmap.data(), &s)))
    return st;
  return dictproj_layer_upload_bitmap(pptr.data(), codes.data(), scales.data(), bitmap.data(), s, k, d_out, out);
}

int dictproj_layer_upload_blocks(const uint32_t* blk_ptr, const uint16_t* blk_idx, const uint8_t* codes,
                                 const uint8_t* scales, float s_C, int k, int d_out, dictproj_layer** out) {
  clear_error();
  if (!blk_ptr || !blk_idx || !codes || !scales || !out) return fail(DICTPROJ_ERR_NULL, "layer_upload_blocks: NULL pointer");
  *out = nullptr;
  if (k <= 0 || k % 16 || k > 65535 || d_out <= 0)
    return fail(DICTPROJ_ERR_SHAPE, "layer_upload_blocks: need 0 < k <= 65535, k %% 16 == 0, d_out > 0 (got k=%d d_out=%d)", k, d_out);
  if (!(s_C > 0.0f) || !std::isfinite(s_C)) return fail(DICTPROJ_ERR_VALUE, "layer_upload_blocks: s_C must be finite and > 0");
  if (blk_ptr[0] != 0) return fail(DICTPROJ_ERR_RANGE, "layer_upload_blocks: blk_ptr[0] must be 0");
  const int nb_max = k / 16;
  for (int o = 0; o < d_out; ++o) {
    if (blk_ptr[o + 1] < blk_ptr[o] || blk_ptr[o + 1] - blk_ptr[o] > (uint32_t)nb_max)
      return fail(DICTPROJ_ERR_RANGE, "layer_upload_blocks: column %d has a bad block count", o);
    for (uint32_t b = blk_ptr[o]; b < blk_ptr[o + 1]; ++b)
      if (blk_idx[b] >= nb_max || (b > blk_ptr[o] && blk_idx[b] <= blk_idx[b - 1]))
        return fail(DICTPROJ_ERR_RANGE, "layer_upload_blocks: column %d block numbers not ascending below k/16", o);
  }
  int st;
  dictproj_layer* l = nullptr;
  if ((st = new_index_layer(k, d_out, s_C, DICTPROJ_IFMT_BLOCKS, &l))) return st;
  const size_t nb = blk_ptr[d_out];
  l->nblk = nb;
  l->total = nb * 16;
  l->nnz_total = nb * 16;
  cudaError_t e;
  if ((e = dmalloc((void**)&l->blk_ptr, (d_out + 1) * sizeof(uint32_t) + 16)) ||
      (e = dmalloc((void**)&l->blk_idx, nb * sizeof(uint16_t) + 16)) || (e = dmalloc((void**)&l->codes, nb * 8 + 16)) ||
      (e = dmalloc((void**)&l->scales, nb + 16))) {
    dictproj_free_layer(l);
    cudaGetLastError();
    return fail(DICTPROJ_ERR_OOM, "layer_upload_blocks: device allocation failed (%s)", cudaGetErrorName(e));
  }
  if ((e = h2d(l->blk_ptr, blk_ptr, (d_out + 1) * sizeof(uint32_t))) ||
      (e = h2d(l->blk_idx, blk_idx, nb * sizeof(uint16_t))) || (e = h2d(l->codes, codes, nb * 8)) ||
      (e = h2d(l->scales, scales, nb))) {
    dictproj_free_layer(l);
    cudaGetLastError();
    return cuda_fail(e, "layer_upload_blocks: copy to device");
  }
  *out = l;
  return DICTPROJ_OK;
}

int dictproj_pack_layer_blocks(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                               dictproj_layer** out) {
  clear_error();
  if (!col_ptr || !out) return fail(DICTPROJ_ERR_NULL, "pack_layer_blocks: NULL pointer");
  *out = nullptr;
  if (k <= 0 || k % 16 || d_out <= 0) return fail(DICTPROJ_ERR_SHAPE, "pack_layer_blocks: k must be a positive multiple of 16");
  const size_t nz = (size_t)col_ptr[d_out];
  std::vector<uint32_t> bptr;
  std::vector<uint16_t> bidx;
  std::vector<uint8_t> codes, scales;
  try {
    bptr.resize(d_out + 1);
    bidx.resize(nz / 16 + 1);
    codes.resize(nz / 2 + 1);
    scales.resize(nz / 16 + 1);
  } catch (...) {
    return fail(DICTPROJ_ERR_OOM, "pack_layer_blocks: host allocation failed");
  }
  float s = 0.f;
  int st;
  if ((st = pack_layer_blocks_host(col_ptr, atom_idx, vals, k, d_out, bptr.data(), bidx.data(), codes.data(),
                                   scales.data(), &s)))
    return st;
  return dictproj_layer_upload_blocks(bptr.data(), bidx.data(), codes.data(), scales.data(), s, k, d_out, out);
}

int dictproj_layer_index_format(const dictproj_layer* l, int* ifmt) {
  clear_error();
  if (!l || !ifmt) return fail(DICTPROJ_ERR_NULL, "layer_index_format: NULL pointer");
  *ifmt = l->ifmt;
  return DICTPROJ_OK;
}

int dictproj_layer_export_bitmap(const dictproj_layer* l, uint32_t* pcol_ptr, uint8_t* codes, uint8_t* scales,
                                 uint32_t* bitmap, float* s_C) {
  clear_error();
  if (!l || !pcol_ptr || !codes || !scales || !bitmap || !s_C) return fail(DICTPROJ_ERR_NULL, "layer_export_bitmap: NULL pointer");
  if (l->ifmt != DICTPROJ_IFMT_BITMAP) return fail(DICTPROJ_ERR_UNSUPPORTED, "layer_export_bitmap: not a bitmap layer");
  const size_t T = l->total;
  cudaError_t e;
  if ((e = cudaMemcpy(pcol_ptr, l->col_ptr, (l->d_out + 1) * sizeof(uint32_t), cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(codes, l->codes, T / 2, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(scales, l->scales, T / 16, cudaMemcpyDeviceToHost)) ||
      (e = cudaMemcpy(bitmap, l->bitmap, (size_t)l->d_out * l->words * sizeof(uint32_t), cudaMemcpyDeviceToHost)))
    return cuda_fail(e, "layer_export_bitmap");
  *s_C = l->s;
  return DICTPROJ_OK;
}

int dictproj_layer_export_blocks(const dictproj_layer* l, uint32_t* blk_ptr, uint16_t* blk_idx, uint8_t* codes,
                                 uint8_t* scales, float* s_C) {
  clear_error();
  if (!l || !blk_ptr || !blk_idx || !codes || !scales || !s_C) return fail(DICTPROJ_ERR_NULL, "layer_export_blocks: NULL pointer");
  if (l->ifmt != DICTPROJ_IFMT_BLOCKS) return fail(DICTPROJ_ERR_UNSUPPORTED, "layer_export_blocks: not a block layer");
  const size_t nb = l->nblk;
  cudaError_t e;
  if ((e = cudaMemcpy(blk_ptr, l->blk_ptr, (l->d_out + 1) * sizeof(uint32_t), cudaMemcpyDeviceToHost)) ||
      (nb && (e = cudaMemcpy(blk_idx, l->blk_idx, nb * sizeof(uint16_t), cudaMemcpyDeviceToHost))) ||
      (nb && (e = cudaMemcpy(codes, l->codes, nb * 8, cudaMemcpyDeviceToHost))) ||
      (nb && (e = cudaMemcpy(scales, l->scales, nb, cudaMemcpyDeviceToHost))))
    return cuda_fail(e, "layer_export_blocks");
  *s_C = l->s;
  return DICTPROJ_OK;
}

int dictproj_group_info(const dictproj_group* g, int* d_in, int* k, int* max_tokens) {
  clear_error();
  if (!g) return fail(DICTPROJ_ERR_NULL, "group_info: NULL handle");
  if (d_in) *d_in = g->d_in;
  if (k) *k = g->k;
  if (max_tokens) *max_tokens = g->max_tokens;
  return DICTPROJ_OK;
}

int dictproj_layer_info(const dictproj_layer* l, int* k, int* d_out, size_t* total, size_t* nnz_total) {
  clear_error();
  if (!l) return fail(DICTPROJ_ERR_NULL, "layer_info: NULL handle");
  if (k) *k = l->k;
  if (d_out) *d_out = l->d_out;
  if (total) *total = l->total;
  if (nnz_total) *nnz_total = l->nnz_total;
  return DICTPROJ_OK;
}

// The two-kernel decode path of one call (stages: bit 0 the dictionary kernel,
// bit 1 the coefficient kernel).
static int launch_split_decode(int n, const dictproj_group* const* groups, const dictproj_layer* const* layers,
                               const __half* const* xs, float* const* zs, const DictPlan* plans, int M, int mp,
                               __half* const* ys, cudaStream_t s, int stages, const char* who) {
  int ns[kDecodeMaxBatch];
  for (int i = 0; i < n; ++i) ns[i] = plans[i].slices;
  cudaError_t e;
  char what[96];
  if ((stages & 1) && (e = launch_dict_decode_batch(n, groups, xs, M, mp, zs, plans, s)) != cudaSuccess) {
    std::snprintf(what, sizeof what, "%s: dictionary stage launch", who);
    return cuda_fail(e, what);
  }
  if ((stages & 2) && (e = launch_coeff_decode_batch(n, layers, zs, ns, M, mp, ys, s)) != cudaSuccess) {
    std::snprintf(what, sizeof what, "%s: coefficient stage launch", who);
    return cuda_fail(e, what);
  }
  return DICTPROJ_OK;
}

int dictproj_forward_path(const void* X, int M, const dictproj_layer* layer, const dictproj_group* group,
                          void* Y, void* stream, int path) {
  clear_error();
  if (!X || !Y || !layer || !group) return fail(DICTPROJ_ERR_NULL, "forward: NULL pointer");
  if (M < 1 || M > group->max_tokens)
    return fail(DICTPROJ_ERR_RANGE, "forward: M=%d outside [1, %d]", M, group->max_tokens);
  if (layer->k != group->k) return fail(DICTPROJ_ERR_MISMATCH, "forward: layer k=%d != group k=%d", layer->k, group->k);
  if (layer->device != group->device)
    return fail(DICTPROJ_ERR_MISMATCH, "forward: layer on device %d, group on device %d", layer->device, group->device);
  if (((uintptr_t)X & 15) || ((uintptr_t)Y & 15)) return fail(DICTPROJ_ERR_ALIGN, "forward: X and Y must be 16-byte aligned");
  if (path < DICTPROJ_PATH_AUTO || path > DICTPROJ_PATH_PREFILL) return fail(DICTPROJ_ERR_RANGE, "forward: bad path %d", path);
  if (path == DICTPROJ_PATH_DECODE && M > kDecodeMaxTokens)
    return fail(DICTPROJ_ERR_UNSUPPORTED, "forward: decode path takes M <= %d (got %d)", kDecodeMaxTokens, M);
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "forward: cudaGetDevice");
  if (dev != group->device)
    return fail(DICTPROJ_ERR_MISMATCH, "forward: current device %d, handles on device %d", dev, group->device);
  cudaStream_t s = (cudaStream_t)stream;
  const __half* x = static_cast<const __half*>(X);
  __half* y = static_cast<__half*>(Y);
  const bool decode = path == DICTPROJ_PATH_DECODE || (path == DICTPROJ_PATH_AUTO && M <= kDecodeMaxTokens);
  const DictPlan plan = dict_plan(group->d_in, group->k, group->n_sm, M < kDecodeMaxTokens ? M : kDecodeMaxTokens, false);
  if (decode) {
    const int mp = decode_mp(M);
    FusedLaunchPlan fp;
    if (use_fused(1, &group, &layer, &x, M, dev, &fp)) {
      if ((e = launch_fused(1, &group, &layer, &x, &y, M, fp, kWaitLimitCycles, s)) != cudaSuccess)
        return cuda_fail(e, "forward: fused decode launch");
      return DICTPROJ_OK;
    }
    if (g_decode_kernels.load(std::memory_order_relaxed) == DICTPROJ_DECODE_FUSED)
      return fail(DICTPROJ_ERR_UNSUPPORTED, "forward: the fused decode kernel does not serve this call "
                                            "(k > 8192 or its shared-memory plan does not fit)");
    if (layer->cfmt != DICTPROJ_CFMT_NVFP4)
      return fail(DICTPROJ_ERR_UNSUPPORTED,
                  "forward: FP16 / FP8 / INT8 coefficients are decoded by the fused kernel only (k <= 8192, Z "
                  "within shared memory); this call falls outside it");
    if (layer->ifmt != DICTPROJ_IFMT_U8 && !index_smem_fits(group->k, mp, dev))
      return fail(DICTPROJ_ERR_UNSUPPORTED,
                  "forward: the bitmap / block decode stages k * %d floats of Z in shared memory; k=%d does not fit "
                  "at M=%d", mp, group->k, M);
    if (layer->ifmt == DICTPROJ_IFMT_U8 && !coeff_smem_fits(group->k, mp, dev))
      return fail(DICTPROJ_ERR_UNSUPPORTED,
                  "forward: the decode path stages (k + 256) * %d floats of Z in shared memory; k=%d does not fit "
                  "at M=%d", mp, group->k, M);
    float* z = group->z32;
    return launch_split_decode(1, &group, &layer, &x, &z, &plan, M, mp, &y, s, 3, "forward");
  }
  // Prefill: Z = s_D X D^ (fp16) and Y = s_C Z C^ as tensor-core GEMMs, C^ densified first.
  if (layer->d_out > group->cdense_cols)
    return fail(DICTPROJ_ERR_RANGE,
                "forward: prefill needs the group's coefficient scratch for d_out=%d (reserved: %d); call "
                "dictproj_group_reserve_prefill first",
                layer->d_out, group->cdense_cols);
  __half* z = reinterpret_cast<__half*>(group->z16);
  __half* cd = reinterpret_cast<__half*>(group->cdense);
  if ((e = launch_dict_prefill(group, x, M, z, s)) != cudaSuccess)
    return cuda_fail(e, "forward: prefill dictionary stage launch");
  if ((e = launch_densify_coeff(layer, cd, s)) != cudaSuccess)
    return cuda_fail(e, "forward: prefill coefficient densify launch");
  if ((e = launch_coeff_prefill(layer, z, cd, M, y, s)) != cudaSuccess)
    return cuda_fail(e, "forward: prefill coefficient stage launch");
  return DICTPROJ_OK;
}

// stages: bit 0 the dictionary kernel, bit 1 the coefficient kernel of the
// two-kernel decode path (3 = the whole forward, which is the only mask the
// fused kernel and the prefill path take).
static int forward_batch_impl(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                              const dictproj_group* const* groups, void* const* Y, void* stream, int stages) {
  clear_error();
  if (stages < 1 || stages > 3) return fail(DICTPROJ_ERR_RANGE, "forward_batch_stages: stage mask %d not 1, 2 or 3", stages);
  if (!X || !layers || !groups || !Y) return fail(DICTPROJ_ERR_NULL, "forward_batch: NULL array");
  if (n < 1 || n > DICTPROJ_MAX_BATCH)
    return fail(DICTPROJ_ERR_RANGE, "forward_batch: n=%d outside [1, %d]", n, DICTPROJ_MAX_BATCH);
  for (int i = 0; i < n; ++i) {
    if (!X[i] || !Y[i] || !layers[i] || !groups[i]) return fail(DICTPROJ_ERR_NULL, "forward_batch: NULL entry %d", i);
    if (M < 1 || M > groups[i]->max_tokens)
      return fail(DICTPROJ_ERR_RANGE, "forward_batch: M=%d outside [1, %d] for entry %d", M, groups[i]->max_tokens, i);
    if (layers[i]->k != groups[i]->k)
      return fail(DICTPROJ_ERR_MISMATCH, "forward_batch: entry %d layer k=%d != group k=%d", i, layers[i]->k,
                  groups[i]->k);
    if (layers[i]->device != groups[i]->device || groups[i]->device != groups[0]->device)
      return fail(DICTPROJ_ERR_MISMATCH, "forward_batch: entries on different devices");
    if (((uintptr_t)X[i] & 15) || ((uintptr_t)Y[i] & 15))
      return fail(DICTPROJ_ERR_ALIGN, "forward_batch: X and Y must be 16-byte aligned (entry %d)", i);
    for (int j = 0; j < i; ++j)
      if (groups[j] == groups[i]) return fail(DICTPROJ_ERR_MISMATCH, "forward_batch: group of entry %d repeated", i);
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "forward_batch: cudaGetDevice");
  if (dev != groups[0]->device)
    return fail(DICTPROJ_ERR_MISMATCH, "forward_batch: current device %d, handles on device %d", dev, groups[0]->device);
  if (M > kDecodeMaxTokens) {  // prefill: one projection after another
    if (stages != 3) return fail(DICTPROJ_ERR_UNSUPPORTED, "forward_batch_stages: a stage mask needs M <= %d", kDecodeMaxTokens);
    for (int i = 0; i < n; ++i) {
      const int st = dictproj_forward_path(X[i], M, layers[i], groups[i], Y[i], stream, DICTPROJ_PATH_AUTO);
      if (st) return st;
    }
    return DICTPROJ_OK;
  }
  const int mp = decode_mp(M);
  cudaStream_t s = (cudaStream_t)stream;
  {
    const __half* xs[kDecodeMaxBatch];
    __half* ys[kDecodeMaxBatch];
    for (int i = 0; i < n; ++i) {
      xs[i] = static_cast<const __half*>(X[i]);
      ys[i] = static_cast<__half*>(Y[i]);
    }
    FusedLaunchPlan fp;
    if (use_fused(n, groups, layers, xs, M, dev, &fp)) {
      if (stages != 3)
        return fail(DICTPROJ_ERR_UNSUPPORTED, "forward_batch_stages: the fused decode kernel serves this call; it has one stage");
      if ((e = launch_fused(n, groups, layers, xs, ys, M, fp, kWaitLimitCycles, s)) != cudaSuccess)
        return cuda_fail(e, "forward_batch: fused decode launch");
      return DICTPROJ_OK;
    }
    if (g_decode_kernels.load(std::memory_order_relaxed) == DICTPROJ_DECODE_FUSED)
      return fail(DICTPROJ_ERR_UNSUPPORTED, "forward_batch: the fused decode kernel does not serve this call "
                                            "(k > 8192 or its shared-memory plan does not fit)");
  }
  for (int i = 0; i < n; ++i)
    if (layers[i]->cfmt != DICTPROJ_CFMT_NVFP4)
      return fail(DICTPROJ_ERR_UNSUPPORTED, "forward_batch: entry %d has FP16 / FP8 / INT8 coefficients, which only "
                  "the fused kernel decodes, and the batch falls outside it", i);
  for (int i = 0; i < n; ++i)
    if (layers[i]->ifmt == DICTPROJ_IFMT_U8 ? !coeff_smem_fits(groups[i]->k, mp, dev)
                                            : !index_smem_fits(groups[i]->k, mp, dev))
      return fail(DICTPROJ_ERR_UNSUPPORTED,
                  "forward_batch: the decode path stages Z (k=%d atoms x %d floats) in shared memory; entry %d "
                  "does not fit at M=%d", groups[i]->k, mp, i, M);
  DictPlan plans[kDecodeMaxBatch];
  const __half* xs[kDecodeMaxBatch];
  float* zs[kDecodeMaxBatch];
  __half* ys[kDecodeMaxBatch];
  int din[kDecodeMaxBatch], kk[kDecodeMaxBatch];
  for (int i = 0; i < n; ++i) din[i] = groups[i]->d_in, kk[i] = groups[i]->k;
  dict_plan_batch(n, din, kk, groups[0]->n_sm, M, plans);
  for (int i = 0; i < n; ++i) {
    if (plans[i].slices > groups[i]->zslices)  // cannot happen: the scratch holds the slices of J = 1
      return fail(DICTPROJ_ERR_UNSUPPORTED, "forward_batch: plan needs %d Z slices, entry %d holds %d",
                  plans[i].slices, i, groups[i]->zslices);
    xs[i] = static_cast<const __half*>(X[i]);
    zs[i] = groups[i]->z32;
    ys[i] = static_cast<__half*>(Y[i]);
  }
  return launch_split_decode(n, groups, layers, xs, zs, plans, M, mp, ys, s, stages, "forward_batch");
}

int dictproj_forward_batch(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                           const dictproj_group* const* groups, void* const* Y, void* stream) {
  return forward_batch_impl(n, X, M, layers, groups, Y, stream, 3);
}

int dictproj_forward_batch_stages(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                                  const dictproj_group* const* groups, void* const* Y, void* stream, int stages) {
  return forward_batch_impl(n, X, M, layers, groups, Y, stream, stages);
}

int dictproj_decode_batch_plan(int n, const int* d_in, const int* k, const int* d_out, const long long* entries,
                               int M, int n_sm, int* dict_ctas, int* dict_slices, int* coeff_ctas) {
  clear_error();
  if (!d_in || !k || !d_out || !entries || !dict_ctas || !dict_slices || !coeff_ctas)
    return fail(DICTPROJ_ERR_NULL, "decode_batch_plan: NULL pointer");
  if (n < 1 || n > DICTPROJ_MAX_BATCH)
    return fail(DICTPROJ_ERR_RANGE, "decode_batch_plan: n=%d outside [1, %d]", n, DICTPROJ_MAX_BATCH);
  if (M < 1 || M > kDecodeMaxTokens) return fail(DICTPROJ_ERR_RANGE, "decode_batch_plan: M=%d outside [1, %d]", M, kDecodeMaxTokens);
  if (n_sm < 1) return fail(DICTPROJ_ERR_RANGE, "decode_batch_plan: n_sm=%d < 1", n_sm);
  size_t ent[kDecodeMaxBatch];
  int cols[kDecodeMaxBatch];
  for (int i = 0; i < n; ++i) {
    if (d_in[i] < 16 || d_in[i] % 16 || k[i] < 16 || k[i] % 16 || d_out[i] < 1)
      return fail(DICTPROJ_ERR_SHAPE, "decode_batch_plan: entry %d has d_in=%d k=%d d_out=%d", i, d_in[i], k[i], d_out[i]);
    if (entries[i] < 0) return fail(DICTPROJ_ERR_RANGE, "decode_batch_plan: entry %d has %lld entries", i, entries[i]);
    ent[i] = (size_t)entries[i];
    cols[i] = d_out[i];
  }
  DictPlan plans[kDecodeMaxBatch];
  dict_plan_batch(n, d_in, k, n_sm, M, plans);
  int share[kDecodeMaxBatch];
  gather_batch_shares(n, ent, cols, n_sm, share);
  for (int i = 0; i < n; ++i) {
    dict_ctas[i] = (k[i] / 16) * plans[i].slices;
    dict_slices[i] = plans[i].slices;
    const int cols = (d_out[i] + share[i] - 1) / share[i];
    coeff_ctas[i] = (d_out[i] + cols - 1) / cols;
  }
  return DICTPROJ_OK;
}

int dictproj_launch_count(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                          const dictproj_group* const* groups, int* count) {
  clear_error();
  if (!X || !layers || !groups || !count) return fail(DICTPROJ_ERR_NULL, "launch_count: NULL pointer");
  if (n < 1 || n > DICTPROJ_MAX_BATCH) return fail(DICTPROJ_ERR_RANGE, "launch_count: n=%d outside [1, %d]", n, DICTPROJ_MAX_BATCH);
  for (int i = 0; i < n; ++i)
    if (!layers[i] || !groups[i]) return fail(DICTPROJ_ERR_NULL, "launch_count: NULL entry %d", i);
  if (M < 1) return fail(DICTPROJ_ERR_RANGE, "launch_count: M=%d < 1", M);
  if (M > kDecodeMaxTokens) {  // prefill: dictionary GEMM, densify, coefficient GEMM per projection
    *count = 3 * n;
    return DICTPROJ_OK;
  }
  const __half* xs[kDecodeMaxBatch];
  for (int i = 0; i < n; ++i) xs[i] = static_cast<const __half*>(X[i]);
  FusedLaunchPlan fp;
  if (use_fused(n, groups, layers, xs, M, groups[0]->device, &fp)) {
    *count = 1;
    return DICTPROJ_OK;
  }
  bool all_gather = true;
  for (int i = 0; i < n; ++i) all_gather = all_gather && layers[i]->gather_ok;
  *count = 1 + (all_gather ? 1 : n);
  return DICTPROJ_OK;
}

int dictproj_set_decode_kernels(int which) {
  clear_error();
  if (which < DICTPROJ_DECODE_AUTO || which > DICTPROJ_DECODE_SPLIT)
    return fail(DICTPROJ_ERR_RANGE, "set_decode_kernels: unknown value %d", which);
  g_decode_kernels.store(which, std::memory_order_relaxed);
  return DICTPROJ_OK;
}

int dictproj_get_decode_kernels(void) { return g_decode_kernels.load(std::memory_order_relaxed); }

int dictproj_forward(const void* X, int M, const dictproj_layer* layer, const dictproj_group* group, void* Y,
                     void* stream) {
  return dictproj_forward_path(X, M, layer, group, Y, stream, DICTPROJ_PATH_AUTO);
}

int dictproj_dictionary_stage(const void* X, int M, const dictproj_group* group, float* Z, void* stream) {
  clear_error();
  if (!X || !group || !Z) return fail(DICTPROJ_ERR_NULL, "dictionary_stage: NULL pointer");
  if (M < 1 || M > group->max_tokens) return fail(DICTPROJ_ERR_RANGE, "dictionary_stage: M=%d outside [1, %d]", M, group->max_tokens);
  if (M > kDecodeMaxTokens) return fail(DICTPROJ_ERR_UNSUPPORTED, "dictionary_stage: M must be <= %d", kDecodeMaxTokens);
  if (((uintptr_t)X & 15) || ((uintptr_t)Z & 15)) return fail(DICTPROJ_ERR_ALIGN, "dictionary_stage: X and Z must be 16-byte aligned");
  const DictPlan plan = dict_plan(group->d_in, group->k, group->n_sm, M, true);  // Z written complete
  cudaError_t e = launch_dict_decode(group, static_cast<const __half*>(X), M, decode_mp(M), Z, plan, (cudaStream_t)stream);
  return e == cudaSuccess ? DICTPROJ_OK : cuda_fail(e, "dictionary_stage: launch");
}

int dictproj_dictionary_stage_prefill(const void* X, int M, const dictproj_group* group, void* Z, void* stream) {
  clear_error();
  if (!X || !group || !Z) return fail(DICTPROJ_ERR_NULL, "dictionary_stage_prefill: NULL pointer");
  if (M < 1) return fail(DICTPROJ_ERR_RANGE, "dictionary_stage_prefill: M=%d < 1", M);
  if (((uintptr_t)X & 15) || ((uintptr_t)Z & 15))
    return fail(DICTPROJ_ERR_ALIGN, "dictionary_stage_prefill: X and Z must be 16-byte aligned");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "dictionary_stage_prefill: cudaGetDevice");
  if (dev != group->device)
    return fail(DICTPROJ_ERR_MISMATCH, "dictionary_stage_prefill: current device %d, group on device %d", dev,
                group->device);
  e = launch_dict_prefill(group, static_cast<const __half*>(X), M, static_cast<__half*>(Z), (cudaStream_t)stream);
  return e == cudaSuccess ? DICTPROJ_OK : cuda_fail(e, "dictionary_stage_prefill: launch");
}

int dictproj_coefficient_stage(const float* Z, int M, const dictproj_layer* layer, void* Y, void* stream) {
  clear_error();
  if (!Z || !layer || !Y) return fail(DICTPROJ_ERR_NULL, "coefficient_stage: NULL pointer");
  if (M < 1) return fail(DICTPROJ_ERR_RANGE, "coefficient_stage: M=%d < 1", M);
  if (M > kDecodeMaxTokens) return fail(DICTPROJ_ERR_UNSUPPORTED, "coefficient_stage: M must be <= %d", kDecodeMaxTokens);
  if (((uintptr_t)Y & 15) || ((uintptr_t)Z & 15)) return fail(DICTPROJ_ERR_ALIGN, "coefficient_stage: Z and Y must be 16-byte aligned");
  if (layer->cfmt != DICTPROJ_CFMT_NVFP4)
    return fail(DICTPROJ_ERR_UNSUPPORTED, "coefficient_stage: NVFP4 coefficients only");
  if (!coeff_smem_fits(layer->k, decode_mp(M), layer->device))
    return fail(DICTPROJ_ERR_UNSUPPORTED, "coefficient_stage: (k + 256) * mp floats of Z do not fit in shared "
                "memory (k=%d, M=%d)", layer->k, M);
  cudaError_t e = launch_coeff_decode(layer, Z, 1, M, decode_mp(M), static_cast<__half*>(Y), (cudaStream_t)stream);
  return e == cudaSuccess ? DICTPROJ_OK : cuda_fail(e, "coefficient_stage: launch");
}

int dictproj_selftest_wait_timeout(long long cycles, void* stream) {
  clear_error();
  if (cycles < 1 || cycles > (1ll << 31))
    return fail(DICTPROJ_ERR_RANGE, "selftest_wait_timeout: cycles=%lld outside [1, 2^31]", cycles);
  int dev, st;
  if ((st = ensure_device(&dev))) return st;
  cudaError_t e = launch_wait_probe(cycles, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_wait_probe_prefill(cycles, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_wait_probe_fused(cycles, (cudaStream_t)stream);
  return e == cudaSuccess ? DICTPROJ_OK : cuda_fail(e, "selftest_wait_timeout: launch");
}

int dictproj_diag_phase_times(unsigned long long* out, int max_ctas, int* n_ctas) {
  clear_error();
  if (!out || !n_ctas) return fail(DICTPROJ_ERR_NULL, "diag_phase_times: NULL pointer");
  if (max_ctas < 1) return fail(DICTPROJ_ERR_RANGE, "diag_phase_times: max_ctas=%d < 1", max_ctas);
  int dev, st;
  if ((st = ensure_device(&dev))) return st;
  cudaError_t e = fused_phase_times(out, max_ctas, n_ctas);
  return e == cudaSuccess ? DICTPROJ_OK : cuda_fail(e, "diag_phase_times");
}

int dictproj_diag_gather_times(unsigned long long* buf, int max_ctas) {
  clear_error();
  if (buf && max_ctas < 1) return fail(DICTPROJ_ERR_RANGE, "diag_gather_times: max_ctas=%d < 1", max_ctas);
  if (((uintptr_t)buf & 7) != 0) return fail(DICTPROJ_ERR_ALIGN, "diag_gather_times: buf must be 8-byte aligned");
  int dev, st;
  if ((st = ensure_device(&dev))) return st;
  cudaError_t e = set_gather_times(buf, max_ctas);
  return e == cudaSuccess ? DICTPROJ_OK : cuda_fail(e, "diag_gather_times");
}

int dictproj_check(void* stream) {
  clear_error();
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "check: stream synchronize");
  unsigned int word = 0;
  if ((e = take_decode_error(&word)) != cudaSuccess) return cuda_fail(e, "check: read error word");
  unsigned int word2 = 0;
  if ((e = take_prefill_error(&word2)) != cudaSuccess) return cuda_fail(e, "check: read error word");
  word |= word2;
  if ((e = take_fused_error(&word2)) != cudaSuccess) return cuda_fail(e, "check: read error word");
  word |= word2;
  if (word) return fail(DICTPROJ_ERR_TIMEOUT, "check: a bounded device wait gave up (error word 0x%x)", word);
  return DICTPROJ_OK;
}

}  // extern "C"
