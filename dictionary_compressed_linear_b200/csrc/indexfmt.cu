// Coefficient-support index formats other than the u8 segment-relative index:
//
//   bitmap (the review's Eq. (12), case a = 0, h = 1, "From retained values to
//     measured decoding"): column o keeps a k-bit mask, uint32[d_out][ceil(k/32)];
//     its set bits, ascending, are the column's stored entries in storage order.
//     Values, padding, block scales and s_C are exactly those of the u8 layout.
//   blocks (block-structured support, the review's "Let the accelerator
//     constrain the support"): every kept support unit is an aligned block of 16
//     consecutive atoms, one uint16 block number per block; a block is exactly
//     one NVFP4 block (16 values, one E4M3 scale).
//
// Decode (M <= 8): the dictionary stage is the shared k_dict_decode; the
// coefficient stage is one of the kernels below, chained with programmatic
// dependent launch. Prefill: a densify kernel per format feeds the same tcgen05
// GEMM as the u8 layout.
//
//   k_coeff_blocks   one warp per column, lanes over its blocks: the 16 Z rows of
//                    a block are 4 aligned float4 loads (no segment logic, no
//                    scattered gathers), 16 fp32 FMAs, one scale per block.
//   k_coeff_bitmap   one warp per column, lanes over its 32-atom words: a warp
//                    scan of the words' popcounts gives each lane the storage
//                    position of its first entry; the lane walks its set bits
//                    (atom = 32*word + bit) with the values in storage order.
//   k_densify_*      one warp per column builds the fp16 row (E2M1 x E4M3 is
//                    exact in fp16) in shared memory, then writes it with 16-B
//                    stores.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {
namespace {

constexpr int kIdxWarps = 32;  // warps per CTA of the decode coefficient kernels

__device__ __forceinline__ void sts_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
constexpr int kBlkRounds = 4;  // blocks per lane whose loads are in flight together

// Z = the sum of the dictionary stage's slices (fixed order) into shared memory.
template <int MP>
__device__ __forceinline__ void stage_z_sum(float* zs, const float* __restrict__ Zpart, int nslices, int k) {
  const int n = k * MP;  // a multiple of 16
  for (int i = threadIdx.x * 4; i < n; i += blockDim.x * 4) {
    float4 a = *reinterpret_cast<const float4*>(Zpart + i);
    for (int sl = 1; sl < nslices; ++sl) {
      const float4 b = *reinterpret_cast<const float4*>(Zpart + (size_t)sl * n + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    *reinterpret_cast<float4*>(zs + i) = a;
  }
}

template <int MP>
__device__ __forceinline__ void warp_sum_store(float acc[MP], int lane, int M, int o, int d_out, float s_C,
                                               __half* __restrict__ Y) {
#pragma unroll
  for (int m = 0; m < MP; ++m) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
  }
  if (lane == 0) {
#pragma unroll
    for (int m = 0; m < MP; ++m)
      if (m < M) Y[(size_t)m * d_out + o] = __float2half_rn(acc[m] * s_C);
  }
}

// ---- block-structured support ---------------------------------------------------------
// The 16 values of block b times the rows Z[16*blk .. 16*blk+15] (MP tokens each),
// unscaled.
template <int MP>
__device__ __forceinline__ void block_dot(float out[MP], const float* zrow, uint2 cw) {
  uint32_t f[8];
  e2m1x8_to_f16x2x4(cw.x, f);
  e2m1x8_to_f16x2x4(cw.y, f + 4);
#pragma unroll
  for (int m = 0; m < MP; ++m) out[m] = 0.f;
  if constexpr (MP == 1) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 z = *reinterpret_cast<const float4*>(zrow + 4 * q);
      const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&f[2 * q]));
      const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&f[2 * q + 1]));
      a0 = fmaf(z.x, v0.x, a0);
      a1 = fmaf(z.y, v0.y, a1);
      a0 = fmaf(z.z, v1.x, a0);
      a1 = fmaf(z.w, v1.y, a1);
    }
    out[0] = a0 + a1;
  } else {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[p]));
#pragma unroll
      for (int m = 0; m < MP; m += 4) {
        const float4 za = *reinterpret_cast<const float4*>(zrow + (2 * p) * MP + m);
        const float4 zb = *reinterpret_cast<const float4*>(zrow + (2 * p + 1) * MP + m);
        out[m] = fmaf(za.x, v.x, fmaf(zb.x, v.y, out[m]));
        if (m + 1 < MP) out[m + 1] = fmaf(za.y, v.x, fmaf(zb.y, v.y, out[m + 1]));
        if (m + 2 < MP) out[m + 2] = fmaf(za.z, v.x, fmaf(zb.z, v.y, out[m + 2]));
        if (m + 3 < MP) out[m + 3] = fmaf(za.w, v.x, fmaf(zb.w, v.y, out[m + 3]));
      }
    }
  }
}

template <int MP>
__device__ __forceinline__ void block_dot2(float out[MP], const float* zrow, uint2 cw) {
  // MP == 2: rows of two tokens; pairs of float4 hold two atoms each
  uint32_t f[8];
  e2m1x8_to_f16x2x4(cw.x, f);
  e2m1x8_to_f16x2x4(cw.y, f + 4);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[p]));
    const float4 z = *reinterpret_cast<const float4*>(zrow + 4 * p);  // atoms 2p, 2p+1 x tokens 0, 1
    a0 = fmaf(z.x, v.x, fmaf(z.z, v.y, a0));
    a1 = fmaf(z.y, v.x, fmaf(z.w, v.y, a1));
  }
  out[0] = a0;
  out[1] = a1;
}

template <int MP>
__global__ void __launch_bounds__(kIdxWarps * 32, 1)
    k_coeff_blocks(const uint32_t* __restrict__ blk_ptr, const uint16_t* __restrict__ blk_idx,
                   const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, float s_C, int k,
                   int d_out, int cols_per_cta, const float* __restrict__ Zpart, int nslices, int M,
                   __half* __restrict__ Y) {
  extern __shared__ __align__(16) float zsb[];  // [k][MP]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o0 = blockIdx.x * cols_per_cta, o1 = min(d_out, o0 + cols_per_cta);
  if (threadIdx.x == 0 && o0 < o1) {  // bulk L2 prefetch of this CTA's blocks
    const size_t b0 = blk_ptr[o0], b1 = blk_ptr[o1];
    prefetch_l2_range(blk_idx, 2 * b0, 2 * b1);
    prefetch_l2_range(codes, 8 * b0, 8 * b1);
    prefetch_l2_range(scales, b0, b1);
  }
  trigger_dependents();
  grid_dependency_wait();  // Z comes from the dictionary stage
  stage_z_sum<MP>(zsb, Zpart, nslices, k);
  __syncthreads();
  for (int o = o0 + warp; o < o1; o += kIdxWarps) {
    const uint32_t b0 = blk_ptr[o], b1 = blk_ptr[o + 1];
    float acc[MP];
#pragma unroll
    for (int m = 0; m < MP; ++m) acc[m] = 0.f;
    for (uint32_t base = b0; base < b1; base += 32 * kBlkRounds) {
      uint32_t bi[kBlkRounds], sb[kBlkRounds];
      uint2 cw[kBlkRounds];
#pragma unroll
      for (int r = 0; r < kBlkRounds; ++r) {  // every load of the rounds first
        const uint32_t b = base + 32 * r + lane;
        bi[r] = 0;
        sb[r] = 0;
        cw[r] = make_uint2(0, 0);
        if (b < b1) {
          bi[r] = blk_idx[b];
          cw[r] = *reinterpret_cast<const uint2*>(codes + 8 * (size_t)b);
          sb[r] = scales[b];
        }
      }
#pragma unroll
      for (int r = 0; r < kBlkRounds; ++r) {
        if (base + 32 * r + lane < b1) {
          float s[MP];
          if constexpr (MP == 2) block_dot2<MP>(s, zsb + (size_t)bi[r] * 16 * MP, cw[r]);
          else block_dot<MP>(s, zsb + (size_t)bi[r] * 16 * MP, cw[r]);
          const float sc = e4m3_to_f32_int(sb[r]);
#pragma unroll
          for (int m = 0; m < MP; ++m) acc[m] = fmaf(s[m], sc, acc[m]);
        }
      }
    }
    warp_sum_store<MP>(acc, lane, M, o, d_out, s_C, Y);
  }
}

// ---- bitmap ------------------------------------------------------------------------------
template <int MP>
__global__ void __launch_bounds__(kIdxWarps * 32, 1)
    k_coeff_bitmap(const uint32_t* __restrict__ col_ptr, const uint32_t* __restrict__ bitmap, int words,
                   const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, float s_C, int k, int d_out,
                   int cols_per_cta, const float* __restrict__ Zpart, int nslices, int M, __half* __restrict__ Y) {
  extern __shared__ __align__(16) float zsm[];  // [k][MP]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o0 = blockIdx.x * cols_per_cta, o1 = min(d_out, o0 + cols_per_cta);
  if (threadIdx.x == 0 && o0 < o1) {  // bulk L2 prefetch of this CTA's columns
    const size_t e0 = col_ptr[o0], e1 = col_ptr[o1];
    prefetch_l2_range(bitmap, 4 * (size_t)o0 * words, 4 * (size_t)o1 * words);
    prefetch_l2_range(codes, e0 >> 1, e1 >> 1);
    prefetch_l2_range(scales, e0 >> 4, e1 >> 4);
  }
  trigger_dependents();
  grid_dependency_wait();
  stage_z_sum<MP>(zsm, Zpart, nslices, k);
  __syncthreads();
  for (int o = o0 + warp; o < o1; o += kIdxWarps) {
    const uint32_t cb = col_ptr[o];
    const uint32_t* row = bitmap + (size_t)o * words;
    float acc[MP];
#pragma unroll
    for (int m = 0; m < MP; ++m) acc[m] = 0.f;
    uint32_t before = 0;  // stored entries of the column's earlier rounds
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t bits = w < words ? row[w] : 0u;
      const int n = __popc(bits);
      int incl = n;  // inclusive scan of the popcounts over the lanes
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      uint32_t e = cb + before + (uint32_t)(incl - n);  // storage position of this lane's first entry
      before += (uint32_t)__shfl_sync(0xffffffffu, incl, 31);
      while (bits) {
        const uint32_t j = (uint32_t)(__ffs(bits) - 1);
        bits &= bits - 1u;
        const uint32_t atom = 32u * (uint32_t)w + j;
        const uint32_t nib = ((uint32_t)codes[e >> 1] >> (4 * (e & 1u))) & 0xFu;
        const float v = __half2float(__ushort_as_half((unsigned short)(e2m1x2_to_f16x2(nib) & 0xFFFFu))) *
                        e4m3_to_f32_int(scales[e >> 4]);
        const float* zr = zsm + (size_t)atom * MP;
#pragma unroll
        for (int m = 0; m < MP; ++m) acc[m] = fmaf(zr[m], v, acc[m]);
        ++e;
      }
    }
    warp_sum_store<MP>(acc, lane, M, o, d_out, s_C, Y);
  }
}

// ---- prefill densify -----------------------------------------------------------------------
// Cd[o][0:k] fp16: the column's values at their atoms, zeros elsewhere.
constexpr int kDensifyWarps = 8;

__global__ void __launch_bounds__(kDensifyWarps * 32)
    k_densify_blocks(const uint32_t* __restrict__ blk_ptr, const uint16_t* __restrict__ blk_idx,
                     const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int k, int d_out,
                     __half* __restrict__ cd) {
  extern __shared__ __align__(16) uint8_t dsb[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * kDensifyWarps + warp;
  grid_dependency_wait();  // Cd may still be read by the previous coefficient GEMM
  if (o >= d_out) return;
  const uint32_t rbase = smem_u32(dsb) + (uint32_t)warp * (uint32_t)k * 2u;
  for (int c = lane; c < k / 8; c += 32) sts_v4(rbase + 16 * c, 0, 0, 0, 0);
  __syncwarp();
  const uint32_t b0 = blk_ptr[o], b1 = blk_ptr[o + 1];
  for (uint32_t b = b0 + lane; b < b1; b += 32) {
    const uint32_t blk = blk_idx[b];
    const uint2 cw = *reinterpret_cast<const uint2*>(codes + 8 * (size_t)b);
    const uint32_t sv = dup_lo(e4m3x2_to_f16x2(scales[b]));
    uint32_t f[8];
    e2m1x8_to_f16x2x4(cw.x, f);
    e2m1x8_to_f16x2x4(cw.y, f + 4);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = hmul2_u32(f[i], sv);  // E2M1 x E4M3 is exact in fp16
    const uint32_t a = rbase + 32u * blk;  // 16 halves = 32 bytes
    sts_v4(a, f[0], f[1], f[2], f[3]);
    sts_v4(a + 16, f[4], f[5], f[6], f[7]);
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(cd + (size_t)o * k);
  for (int c = lane; c < k / 8; c += 32) dst[c] = lds_u32x4(rbase + 16 * c);
}

__global__ void __launch_bounds__(kDensifyWarps * 32)
    k_densify_bitmap(const uint32_t* __restrict__ col_ptr, const uint32_t* __restrict__ bitmap, int words,
                     const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int k, int d_out,
                     __half* __restrict__ cd) {
  extern __shared__ __align__(16) uint8_t dsm2[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * kDensifyWarps + warp;
  grid_dependency_wait();
  if (o >= d_out) return;
  __half* row = reinterpret_cast<__half*>(dsm2) + (size_t)warp * k;
  const uint32_t rbase = smem_u32(row);
  for (int c = lane; c < k / 8; c += 32) sts_v4(rbase + 16 * c, 0, 0, 0, 0);
  __syncwarp();
  const uint32_t cb = col_ptr[o];
  const uint32_t* brow = bitmap + (size_t)o * words;
  uint32_t before = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    uint32_t bits = w < words ? brow[w] : 0u;
    const int n = __popc(bits);
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    uint32_t e = cb + before + (uint32_t)(incl - n);
    before += (uint32_t)__shfl_sync(0xffffffffu, incl, 31);
    while (bits) {
      const uint32_t j = (uint32_t)(__ffs(bits) - 1);
      bits &= bits - 1u;
      const uint32_t nib = ((uint32_t)codes[e >> 1] >> (4 * (e & 1u))) & 0xFu;
      const uint32_t h = hmul2_u32(e2m1x2_to_f16x2(nib), dup_lo(e4m3x2_to_f16x2(scales[e >> 4])));
      row[32u * (uint32_t)w + j] = __ushort_as_half((unsigned short)(h & 0xFFFFu));
      ++e;
    }
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(cd + (size_t)o * k);
  for (int c = lane; c < k / 8; c += 32) dst[c] = lds_u32x4(rbase + 16 * c);
}

cudaError_t launch_pdl_c(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, void** args) {
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

template <int MP>
cudaError_t launch_index_mp(const dictproj_layer* l, const float* Zpart, int nslices, int M, __half* Y,
                            cudaStream_t stream) {
  const int grid = std::max(1, std::min(l->n_sm, l->d_out));
  int cpc = (l->d_out + grid - 1) / grid;
  const size_t smem = (size_t)l->k * MP * sizeof(float);
  float s = l->s;
  int k = l->k, d_out = l->d_out;
  if (l->ifmt == DICTPROJ_IFMT_BLOCKS) {
    const void* fn = (const void*)k_coeff_blocks<MP>;
    void* args[] = {(void*)&l->blk_ptr, (void*)&l->blk_idx, (void*)&l->codes, (void*)&l->scales, &s, &k, &d_out,
                    &cpc, (void*)&Zpart, &nslices, &M, &Y};
    return launch_pdl_c(fn, dim3(grid), dim3(kIdxWarps * 32), smem, stream, args);
  }
  const void* fn = (const void*)k_coeff_bitmap<MP>;
  int words = l->words;
  void* args[] = {(void*)&l->col_ptr, (void*)&l->bitmap, &words, (void*)&l->codes, (void*)&l->scales, &s, &k, &d_out,
                  &cpc, (void*)&Zpart, &nslices, &M, &Y};
  return launch_pdl_c(fn, dim3(grid), dim3(kIdxWarps * 32), smem, stream, args);
}

}  // namespace

cudaError_t prepare_index_kernels(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  const void* fns[] = {(const void*)k_coeff_blocks<1>, (const void*)k_coeff_blocks<2>, (const void*)k_coeff_blocks<4>,
                       (const void*)k_coeff_blocks<8>, (const void*)k_coeff_bitmap<1>, (const void*)k_coeff_bitmap<2>,
                       (const void*)k_coeff_bitmap<4>, (const void*)k_coeff_bitmap<8>, (const void*)k_densify_blocks,
                       (const void*)k_densify_bitmap};
  for (const void* fn : fns)
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)) != cudaSuccess) return e;
  return cudaSuccess;
}

bool index_smem_fits(int k, int mp, int device) {
  return (size_t)k * mp * sizeof(float) <= (size_t)smem_optin_of(device);
}

cudaError_t launch_coeff_index(const dictproj_layer* l, const float* Zpart, int nslices, int M, int mp, __half* Y,
                               cudaStream_t stream) {
  switch (mp) {
    case 1: return launch_index_mp<1>(l, Zpart, nslices, M, Y, stream);
    case 2: return launch_index_mp<2>(l, Zpart, nslices, M, Y, stream);
    case 4: return launch_index_mp<4>(l, Zpart, nslices, M, Y, stream);
    default: return launch_index_mp<8>(l, Zpart, nslices, M, Y, stream);
  }
}

cudaError_t launch_densify_index(const dictproj_layer* l, __half* Cd, cudaStream_t stream) {
  const int grid = (l->d_out + kDensifyWarps - 1) / kDensifyWarps;
  const size_t smem = (size_t)kDensifyWarps * l->k * 2;
  int k = l->k, d_out = l->d_out;
  if (l->ifmt == DICTPROJ_IFMT_BLOCKS) {
    void* args[] = {(void*)&l->blk_ptr, (void*)&l->blk_idx, (void*)&l->codes, (void*)&l->scales, &k, &d_out, &Cd};
    return launch_pdl_c((const void*)k_densify_blocks, dim3(grid), dim3(kDensifyWarps * 32), smem, stream, args);
  }
  int words = l->words;
  void* args[] = {(void*)&l->col_ptr, (void*)&l->bitmap, &words, (void*)&l->codes, (void*)&l->scales, &k, &d_out, &Cd};
  return launch_pdl_c((const void*)k_densify_bitmap, dim3(grid), dim3(kDensifyWarps * 32), smem, stream, args);
}

}  // namespace dictproj
