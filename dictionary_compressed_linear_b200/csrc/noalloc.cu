// Decode-path forward that allocates nothing.
//
// Some callers cannot call cudaMalloc when they run a projection: runtimes that
// reserve all device memory up front in their own arena (an allocation at call
// time would fail or fragment it), and code that enqueues work while a stream is
// being captured into a CUDA graph, where allocation calls are not allowed.
// dictproj_forward_noalloc serves them: the caller passes device copies of the
// packed D_g / C_l bytes plus X and Y, all memory it owns, and the Z scratch
// between the two stages lives in the file-scope device array below.
//
// The array is part of the library image, so every GPU that loads the library
// holds it until exit. Its device address is resolved once per device, on the
// first call made with that device current. Every call shares the array: calls
// that overlap on the GPU (different streams, or another thread) race on it and
// must be serialised by the caller. Nothing in it must start at zero: within a
// call the dictionary kernel writes every element the coefficient kernel reads.
#include <mutex>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dictproj.h"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {

// 192 KiB. The coefficient kernel stages (k + 256) * mp floats of Z in shared
// memory, so (k + 256) * mp <= 49152 bounds both that stage and this array.
constexpr int kStaticZFloats = 49152;

static __device__ __align__(256) float g_static_z[kStaticZFloats];

static std::mutex g_static_mu;
static std::vector<float*> g_static_ptr;  // per device

// Device address of g_static_z for the current device (host code cannot use the
// symbol itself: in host code it names a host-side stand-in).
static int static_z(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "forward_noalloc: cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_static_mu);
  if ((int)g_static_ptr.size() <= dev) g_static_ptr.resize(dev + 1, nullptr);
  if (!g_static_ptr[dev]) {
    float* p = nullptr;
    if ((e = cudaGetSymbolAddress((void**)&p, g_static_z)) != cudaSuccess)
      return cuda_fail(e, "forward_noalloc: cudaGetSymbolAddress");
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return DICTPROJ_OK;
}

}  // namespace dictproj

using namespace dictproj;

extern "C" int dictproj_forward_noalloc(const dictproj_device_group* group, const dictproj_device_layer* layer,
                                        const void* X, int M, void* Y, void* stream) {
  clear_error();
  if (!group || !layer || !X || !Y) return fail(DICTPROJ_ERR_NULL, "forward_noalloc: NULL pointer");
  if (!group->codes || !group->scales || !layer->col_ptr || !layer->codes || !layer->scales || !layer->idx ||
      !layer->seg_start)
    return fail(DICTPROJ_ERR_NULL, "forward_noalloc: NULL packed array");
  const int d_in = group->d_in, k = group->k;
  if (d_in <= 0 || d_in % 32 || k <= 0 || k % 16 || k > 65535 || layer->d_out <= 0)
    return fail(DICTPROJ_ERR_SHAPE, "forward_noalloc: need d_in %% 32 == 0, k %% 16 == 0, k <= 65535, d_out > 0 "
                "(got d_in=%d k=%d d_out=%d)", d_in, k, layer->d_out);
  if (layer->k != k) return fail(DICTPROJ_ERR_MISMATCH, "forward_noalloc: layer k=%d != group k=%d", layer->k, k);
  if (M < 1 || M > kDecodeMaxTokens)
    return fail(DICTPROJ_ERR_RANGE, "forward_noalloc: M=%d outside [1, %d]", M, kDecodeMaxTokens);
  const int mp = decode_mp(M);
  if ((size_t)(k + 256) * mp > (size_t)kStaticZFloats)
    return fail(DICTPROJ_ERR_RANGE,
                "forward_noalloc: (k + 256) * mp = (%d + 256) * %d exceeds the static scratch limit of %d floats",
                k, mp, kStaticZFloats);
  if (((uintptr_t)X & 15) || ((uintptr_t)Y & 15))
    return fail(DICTPROJ_ERR_ALIGN, "forward_noalloc: X and Y must be 16-byte aligned");
  // The kernels read the packed arrays with vector loads of up to 16 bytes and
  // prefetch them in 16-byte chunks: every array must start on a 16-byte boundary.
  const void* arrays[] = {group->codes, group->scales, layer->col_ptr, layer->codes,
                          layer->scales, layer->idx, layer->seg_start};
  const char* names[] = {"group codes", "group scales", "layer col_ptr", "layer codes",
                         "layer scales", "layer idx", "layer seg_start"};
  for (int i = 0; i < 7; ++i)
    if ((uintptr_t)arrays[i] & 15)
      return fail(DICTPROJ_ERR_ALIGN, "forward_noalloc: %s must be 16-byte aligned", names[i]);
  if (!(group->s > 0.0f) || !(layer->s > 0.0f)) return fail(DICTPROJ_ERR_VALUE, "forward_noalloc: scales must be > 0");
  int dev, st;
  if ((st = ensure_device(&dev))) return st;
  float* z = nullptr;
  if ((st = static_z(&z))) return st;

  // Views of the caller's buffers (host structs on the stack; no allocation).
  dictproj_group g{};
  g.device = dev;
  g.d_in = d_in;
  g.k = k;
  g.max_tokens = kDecodeMaxTokens;
  g.s = group->s;
  g.codes = const_cast<uint8_t*>(group->codes);
  g.scales = const_cast<uint8_t*>(group->scales);
  dictproj_layer l{};
  l.device = dev;
  l.k = k;
  l.d_out = layer->d_out;
  l.nseg = (k + 255) / 256;
  l.s = layer->s;
  l.col_ptr = const_cast<uint32_t*>(layer->col_ptr);
  l.codes = const_cast<uint8_t*>(layer->codes);
  l.scales = const_cast<uint8_t*>(layer->scales);
  l.idx = const_cast<uint8_t*>(layer->idx);
  l.seg_start = const_cast<uint16_t*>(layer->seg_start);
  // gather_ok stays false: the coefficient stage runs the direct kernel, whose
  // shared memory is only Z

  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  const DictPlan plan = dict_plan(d_in, k, 1, M, true);  // one slice: Z fits the static array
  if ((e = launch_dict_decode(&g, static_cast<const __half*>(X), M, mp, z, plan, s)) != cudaSuccess)
    return cuda_fail(e, "forward_noalloc: dictionary stage launch");
  if ((e = launch_coeff_decode(&l, z, 1, M, mp, static_cast<__half*>(Y), s)) != cudaSuccess)
    return cuda_fail(e, "forward_noalloc: coefficient stage launch");
  return DICTPROJ_OK;
}
