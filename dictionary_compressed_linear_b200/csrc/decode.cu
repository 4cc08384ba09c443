// Decode path (M <= 8 tokens): the two stages of Eq. (1) of the DictLLM
// technical review, Z = X D_g then Y = Z C_l, as two kernels chained with
// programmatic dependent launch.
//
// Stage 1 (dictionary, HBM-bound GEMV over packed NVFP4 D_g).
//   One CTA per tile of 16 atoms; its 8 warps split d_in into 32-element units.
//   Every thread streams 16-byte packed code words of two atoms (rows g, g+8 of
//   a 16x8x16 MMA), converts E2M1 pairs to f16x2 with the hardware cvt, scales
//   them by their E4M3 block scale in fp16 (the product of an E2M1 and an E4M3
//   value is exact in fp16), and feeds mma.sync m16n8k16 with the tokens as the
//   N = 8 dimension (swap-AB), accumulating in fp32. Warp partial sums are
//   reduced in shared memory in a fixed order; Z = s_D * sum, fp32 [k][mp].
//   Packed weights are prefetched (L2 bulk prefetch plus the first register
//   batch) before the grid dependency wait, since no kernel writes them.
//
// Stage 2 (coefficients, sparse gather over column-compressed NVFP4 C_l).
//   Z is staged in shared memory. Each warp takes 4 output columns with 8 lanes
//   per column; a lane processes whole 16-entry blocks (one E4M3 scale each):
//   16 index bytes, 8 code bytes, 1 scale byte. Atom = 256*segment + idx, with
//   the segment tracked incrementally from seg_start. Block sums are scaled by
//   the block scale, lane sums reduced with shuffles, Y = s_C * sum in fp16.
#include <climits>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {

constexpr int kDictWarps = 8;
constexpr int kDictDepth = 4;  // register prefetch depth (iterations)

struct DictUnit {
  uint4 wa, wb;   // 16 code bytes of atoms g and g+8
  uint32_t sa, sb;  // 2 scale bytes each
};

__device__ __forceinline__ void load_unit(DictUnit& u, const uint8_t* c0, const uint8_t* c1,
                                          const uint8_t* s0, const uint8_t* s1, int unit, bool ok) {
  if (ok) {
    u.wa = ld_stream_v4(c0 + (size_t)unit * 16);
    u.wb = ld_stream_v4(c1 + (size_t)unit * 16);
    u.sa = ld_stream_u16(s0 + (size_t)unit * 2);
    u.sb = ld_stream_u16(s1 + (size_t)unit * 2);
  } else {
    u.wa = make_uint4(0, 0, 0, 0);
    u.wb = u.wa;
    u.sa = 0;
    u.sb = 0;
  }
}

__device__ __forceinline__ void dict_unit_mma(float acc[4], const DictUnit& u, const uint4 xv[4]) {
  const uint32_t ha = e4m3x2_to_f16x2(u.sa), hb = e4m3x2_to_f16x2(u.sb);
  const uint32_t wa[4] = {u.wa.x, u.wa.y, u.wa.z, u.wa.w};
  const uint32_t wb[4] = {u.wb.x, u.wb.y, u.wb.z, u.wb.w};
  const uint32_t xw[16] = {xv[0].x, xv[0].y, xv[0].z, xv[0].w, xv[1].x, xv[1].y, xv[1].z, xv[1].w,
                           xv[2].x, xv[2].y, xv[2].z, xv[2].w, xv[3].x, xv[3].y, xv[3].z, xv[3].w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // code word q: elements 8q .. 8q+7 of the unit
    uint32_t fa[4], fb[4];
    e2m1x8_to_f16x2x4(wa[q], fa);
    e2m1x8_to_f16x2x4(wb[q], fb);
    const uint32_t sa = q < 2 ? dup_lo(ha) : dup_hi(ha);  // block 2u for elements 0..15
    const uint32_t sb = q < 2 ? dup_lo(hb) : dup_hi(hb);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      fa[i] = hmul2_u32(fa[i], sa);
      fb[i] = hmul2_u32(fb[i], sb);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // k-slots (2t, 2t+1) <- elements 8q+4h+{0,1}; (2t+8, 2t+9) <- 8q+4h+{2,3}
      const uint32_t a[4] = {fa[2 * h], fb[2 * h], fa[2 * h + 1], fb[2 * h + 1]};
      const uint32_t b[2] = {xw[4 * q + 2 * h], xw[4 * q + 2 * h + 1]};
      mma_16816(acc, a, b);
    }
  }
}

__global__ void __launch_bounds__(kDictWarps * 32)
k_dict_decode(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, float s_D,
              int d_in, const __half* __restrict__ X, int M, int mp, float* __restrict__ Z) {
  constexpr int P = 4 * kDictWarps;
  const int tile = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int p = warp * 4 + tig;
  const int n_units = d_in >> 5;
  const size_t crow = (size_t)(d_in >> 1), srow = (size_t)(d_in >> 4);
  const uint8_t* c0 = codes + (size_t)(tile * 16 + g) * crow;
  const uint8_t* c1 = c0 + 8 * crow;
  const uint8_t* s0 = scales + (size_t)(tile * 16 + g) * srow;
  const uint8_t* s1 = s0 + 8 * srow;

  if (threadIdx.x == 0) {
    prefetch_l2_range(codes, (size_t)tile * 16 * crow, (size_t)(tile + 1) * 16 * crow);
    prefetch_l2_range(scales, (size_t)tile * 16 * srow, (size_t)(tile + 1) * 16 * srow);
  }
  const int iters = (n_units + P - 1) / P;
  DictUnit ring[kDictDepth];
#pragma unroll
  for (int d = 0; d < kDictDepth; ++d) {
    const int u = p + d * P;
    load_unit(ring[d], c0, c1, s0, s1, u, d < iters && u < n_units);
  }
  trigger_dependents();
  grid_dependency_wait();  // X and the Z scratch belong to earlier work on the stream

  const bool xrow = g < M;
  const __half* xr = X + (size_t)g * d_in;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int it0 = 0; it0 < iters; it0 += kDictDepth) {
#pragma unroll
    for (int d = 0; d < kDictDepth; ++d) {
      const int it = it0 + d;
      if (it < iters) {
        const int u = p + it * P;
        uint4 xv[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                       make_uint4(0, 0, 0, 0)};
        if (xrow && u < n_units) {
#pragma unroll
          for (int q = 0; q < 4; ++q) xv[q] = ld_nc_v4(xr + (size_t)u * 32 + q * 8);
        }
        dict_unit_mma(acc, ring[d], xv);
        const int un = p + (it + kDictDepth) * P;
        load_unit(ring[d], c0, c1, s0, s1, un, (it + kDictDepth) < iters && un < n_units);
      }
    }
  }

  __shared__ float red[kDictWarps][16][8];
  red[warp][g][2 * tig] = acc[0];
  red[warp][g][2 * tig + 1] = acc[1];
  red[warp][g + 8][2 * tig] = acc[2];
  red[warp][g + 8][2 * tig + 1] = acc[3];
  __syncthreads();
  if (threadIdx.x < 128) {
    const int a = threadIdx.x >> 3, n = threadIdx.x & 7;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kDictWarps; ++w) s += red[w][a][n];
    if (n < mp) Z[(size_t)(tile * 16 + a) * mp + n] = s * s_D;
  }
}

// ---------------------------------------------------------------------------------
constexpr int kCoeffWarps = 8;
constexpr int kColsPerWarp = 4;
constexpr int kLanesPerCol = 32 / kColsPerWarp;

template <int MP>
__device__ __forceinline__ void fma_z(float blk[MP], const float* z, float v) {
  if constexpr (MP == 1) {
    blk[0] = fmaf(z[0], v, blk[0]);
  } else if constexpr (MP == 2) {
    const float2 t = *reinterpret_cast<const float2*>(z);
    blk[0] = fmaf(t.x, v, blk[0]);
    blk[1] = fmaf(t.y, v, blk[1]);
  } else {
#pragma unroll
    for (int m = 0; m < MP; m += 4) {
      const float4 t = *reinterpret_cast<const float4*>(z + m);
      blk[m] = fmaf(t.x, v, blk[m]);
      blk[m + 1] = fmaf(t.y, v, blk[m + 1]);
      blk[m + 2] = fmaf(t.z, v, blk[m + 2]);
      blk[m + 3] = fmaf(t.w, v, blk[m + 3]);
    }
  }
}

template <int MP>
__global__ void __launch_bounds__(kCoeffWarps * 32)
k_coeff_decode(const uint32_t* __restrict__ col_ptr, const uint8_t* __restrict__ codes,
               const uint8_t* __restrict__ scales, const uint8_t* __restrict__ idx,
               const uint16_t* __restrict__ seg_start, int nseg, float s_C, int k, int d_out,
               const float* __restrict__ Z, int M, __half* __restrict__ Y) {
  extern __shared__ __align__(16) float zs[];  // [k][MP]
  constexpr int kCols = kCoeffWarps * kColsPerWarp;
  const int o0 = blockIdx.x * kCols;
  if (threadIdx.x == 0) {
    const int o1 = min(d_out, o0 + kCols);
    const size_t e0 = col_ptr[o0], e1 = col_ptr[o1];
    prefetch_l2_range(idx, e0, e1);
    prefetch_l2_range(codes, e0 >> 1, e1 >> 1);
    prefetch_l2_range(scales, e0 >> 4, e1 >> 4);
    prefetch_l2_range(seg_start, (size_t)o0 * nseg * 2, (size_t)o1 * nseg * 2);
  }
  trigger_dependents();
  grid_dependency_wait();  // Z comes from the dictionary stage

  for (int i = threadIdx.x * 4; i < k * MP; i += blockDim.x * 4)
    *reinterpret_cast<float4*>(zs + i) = *reinterpret_cast<const float4*>(Z + i);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gl = lane % kLanesPerCol;
  const int o = o0 + warp * kColsPerWarp + lane / kLanesPerCol;
  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.f;
  if (o < d_out) {
    const uint32_t cb = col_ptr[o], ce = col_ptr[o + 1];
    const int nblk = (int)((ce - cb) >> 4);
    const uint16_t* ss = seg_start + (size_t)o * nseg;
    int s = 0;
    int nb = nseg > 1 ? (int)ss[1] : INT_MAX;
    for (int b = gl; b < nblk; b += kLanesPerCol) {
      const int q0 = b << 4;
      const size_t e = cb + (size_t)q0;
      const uint4 iv = ld_stream_v4(idx + e);
      const uint2 cv = ld_stream_v2(codes + (e >> 1));
      const uint32_t scb = ld_stream_u8(scales + (e >> 4));
      while (q0 >= nb) {
        ++s;
        nb = (s + 1 < nseg) ? (int)ss[s + 1] : INT_MAX;
      }
      const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
      const uint32_t cw[2] = {cv.x, cv.y};
      float blk[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) blk[m] = 0.f;
      if (q0 + 15 < nb) {  // the whole block lies in segment s
        const float* zb = zs + (size_t)(s << 8) * MP;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint32_t f[4];
          e2m1x8_to_f16x2x4(cw[j], f);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[i]));
            const int ent = 8 * j + 2 * i;
            const uint32_t a0 = (iw[ent >> 2] >> ((ent & 3) * 8)) & 0xFFu;
            const uint32_t a1 = (iw[(ent + 1) >> 2] >> (((ent + 1) & 3) * 8)) & 0xFFu;
            fma_z<MP>(blk, zb + a0 * MP, v.x);
            fma_z<MP>(blk, zb + a1 * MP, v.y);
          }
        }
      } else {  // the block crosses a segment boundary
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint32_t f[4];
          e2m1x8_to_f16x2x4(cw[j], f);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[i]));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int ent = 8 * j + 2 * i + h;
              const int q = q0 + ent;
              while (q >= nb) {
                ++s;
                nb = (s + 1 < nseg) ? (int)ss[s + 1] : INT_MAX;
              }
              const uint32_t a = ((uint32_t)s << 8) + ((iw[ent >> 2] >> ((ent & 3) * 8)) & 0xFFu);
              fma_z<MP>(blk, zs + (size_t)a * MP, h ? v.y : v.x);
            }
          }
        }
      }
      const float sc = e4m3_to_f32(scb);
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] = fmaf(blk[m], sc, acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) {
#pragma unroll
    for (int off = kLanesPerCol / 2; off > 0; off >>= 1)
      acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
  }
  if (o < d_out && gl == 0) {
#pragma unroll
    for (int m = 0; m < MP; ++m)
      if (m < M) Y[(size_t)m * d_out + o] = __float2half_rn(acc[m] * s_C);
  }
}

// ---------------------------------------------------------------------------------
static cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

int decode_mp(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

size_t coeff_decode_smem(int k, int mp) { return (size_t)k * mp * sizeof(float); }

cudaError_t prepare_decode_kernels(int device) {
  (void)device;
  const int max_smem = 227 * 1024;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_coeff_decode<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_coeff_decode<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_coeff_decode<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_coeff_decode<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem))) return e;
  return cudaSuccess;
}

cudaError_t launch_dict_decode(const dictproj_group* g, const __half* X, int M, int mp, float* Z,
                               cudaStream_t stream) {
  const uint8_t* codes = g->codes;
  const uint8_t* scales = g->scales;
  float s = g->s;
  int d_in = g->d_in;
  void* args[] = {(void*)&codes, (void*)&scales, (void*)&s, (void*)&d_in, (void*)&X,
                  (void*)&M, (void*)&mp, (void*)&Z};
  return launch_pdl((const void*)k_dict_decode, dim3(g->k / 16), dim3(kDictWarps * 32), 0, stream,
                    args);
}

cudaError_t launch_coeff_decode(const dictproj_layer* l, const float* Z, int M, int mp, __half* Y,
                                cudaStream_t stream) {
  const uint32_t* col_ptr = l->col_ptr;
  const uint8_t* codes = l->codes;
  const uint8_t* scales = l->scales;
  const uint8_t* idx = l->idx;
  const uint16_t* ss = l->seg_start;
  int nseg = l->nseg;
  float s = l->s;
  int k = l->k, d_out = l->d_out;
  void* args[] = {(void*)&col_ptr, (void*)&codes, (void*)&scales, (void*)&idx, (void*)&ss,
                  (void*)&nseg, (void*)&s, (void*)&k, (void*)&d_out, (void*)&Z,
                  (void*)&M, (void*)&Y};
  constexpr int kCols = kCoeffWarps * kColsPerWarp;
  const dim3 grid((d_out + kCols - 1) / kCols), block(kCoeffWarps * 32);
  const size_t smem = coeff_decode_smem(k, mp);
  switch (mp) {
    case 1: return launch_pdl((const void*)k_coeff_decode<1>, grid, block, smem, stream, args);
    case 2: return launch_pdl((const void*)k_coeff_decode<2>, grid, block, smem, stream, args);
    case 4: return launch_pdl((const void*)k_coeff_decode<4>, grid, block, smem, stream, args);
    default: return launch_pdl((const void*)k_coeff_decode<8>, grid, block, smem, stream, args);
  }
}

}  // namespace dictproj
