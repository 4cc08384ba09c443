// Decode path (M <= 8 tokens): the two stages of Eq. (1) of the DictLLM
// technical review, Z = X D_g then Y = Z C_l, as two kernels chained with
// programmatic dependent launch. Both issue the reads of their packed weights
// before waiting on the previous kernel (nothing writes weights after upload),
// so weight traffic overlaps the tail of the preceding work on the stream.
//
// Stage 1, dictionary (HBM-bound GEMV over packed NVFP4 D_g), k_dict_decode.
//   One CTA per tile of 8 atoms, 8 warps splitting d_in into 32-element units.
//   Each thread streams 16-byte code words of one atom through a 4-deep register
//   ring (plus a bulk L2 prefetch of the whole tile), converts E2M1 pairs to
//   f16x2 with the hardware cvt, multiplies by the block's E4M3 scale in fp16
//   (an E2M1 x E4M3 product is exact in fp16) and feeds mma.sync m16n8k16 with
//   D as the B operand (N = 8 atoms) and the tokens as A rows, fp32 accumulate.
//   X is staged once in shared memory. Warp partials are summed in a fixed order;
//   Z = s_D * sum as fp32 [k][mp].
//
// Stage 2, coefficients (sparse gather over column-compressed NVFP4 C_l),
// k_coeff_decode.
//   One persistent CTA per SM owns a run of columns balanced by stored entries.
//   The run is cut (on the host, at upload) into chunks of at most 16384 entries
//   of equal per-column padded length. Chunks stream through a two-stage shared
//   memory ring with bulk async copies completing on mbarriers (the first two
//   are issued before the dependency wait). Z is staged in shared memory. Every
//   thread takes a contiguous run of 16-entry blocks (one E4M3 scale each):
//   atom = 256*segment + idx, segment from the column's seg_start row; the block
//   sum is scaled and stored per block; one warp per column then sums the block
//   partials in a fixed order, so results are bit-reproducible.
#include <algorithm>
#include <climits>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {

// =================================================================================
// Stage 1: dictionary
// =================================================================================
constexpr int kDictWarps = 8;
constexpr int kDictDepth = 4;     // register prefetch depth (iterations)
constexpr int kDictAtoms = 8;     // atoms per CTA = MMA N
constexpr size_t kDictXSmemMax = 96 * 1024;

struct DictUnit {
  uint4 w;       // 16 code bytes: 32 elements of this thread's atom
  uint32_t sc;   // the two E4M3 block scales of those 32 elements
};

__device__ __forceinline__ void load_unit(DictUnit& u, const uint8_t* c, const uint8_t* s, int unit, bool ok) {
  if (ok) {
    u.w = ld_stream_v4(c + (size_t)unit * 16);
    u.sc = ld_stream_u16(s + (size_t)unit * 2);
  } else {
    u.w = make_uint4(0, 0, 0, 0);
    u.sc = 0;
  }
}

// One 32-element unit: 8 MMAs of k = 16 (4 elements per thread each).
// B (K x N = d_in-slots x atoms): b0:b1 <- elements 8q+4h+{0,1}, b2:b3 <- 8q+4h+{2,3}.
// A (M x K = tokens x slots): row g (token g) the matching X values, row g+8 zero.
__device__ __forceinline__ void dict_unit_mma(float acc[2][4], const DictUnit& u, const uint32_t xw[16]) {
  const uint32_t h2 = e4m3x2_to_f16x2(u.sc);
  const uint32_t s_lo = dup_lo(h2), s_hi = dup_hi(h2);
  const uint32_t w[4] = {u.w.x, u.w.y, u.w.z, u.w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t f[4];
    e2m1x8_to_f16x2x4(w[q], f);
    const uint32_t sc = q < 2 ? s_lo : s_hi;
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = hmul2_u32(f[i], sc);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a[4] = {xw[4 * q + 2 * h], 0u, xw[4 * q + 2 * h + 1], 0u};
      const uint32_t b[2] = {f[2 * h], f[2 * h + 1]};
      mma_16816(acc[h], a, b);  // two independent accumulation chains
    }
  }
}

template <bool XS>
__global__ void __launch_bounds__(kDictWarps * 32)
k_dict_decode(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, float s_D,
              int d_in, const __half* __restrict__ X, int M, int mp, float* __restrict__ Z) {
  extern __shared__ __align__(16) unsigned char dsmem[];  // X rows, stride d_in + 8 halves
  __shared__ float red[kDictWarps][8][kDictAtoms];
  constexpr int P = 4 * kDictWarps;
  const int tile = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int p = warp * 4 + tig;
  const int n_units = d_in >> 5;
  const size_t crow = (size_t)(d_in >> 1), srow = (size_t)(d_in >> 4);
  const uint8_t* c = codes + (size_t)(tile * kDictAtoms + g) * crow;
  const uint8_t* s = scales + (size_t)(tile * kDictAtoms + g) * srow;

  if (threadIdx.x == 0) {
    prefetch_l2_range(codes, (size_t)tile * kDictAtoms * crow, (size_t)(tile + 1) * kDictAtoms * crow);
    prefetch_l2_range(scales, (size_t)tile * kDictAtoms * srow, (size_t)(tile + 1) * kDictAtoms * srow);
  }
  const int iters = (n_units + P - 1) / P;
  DictUnit ring[kDictDepth];
#pragma unroll
  for (int d = 0; d < kDictDepth; ++d) {
    const int u = p + d * P;
    load_unit(ring[d], c, s, u, d < iters && u < n_units);
  }
  trigger_dependents();
  grid_dependency_wait();  // X and Z belong to earlier work on the stream

  const int xstride = XS ? d_in + 8 : d_in;
  const __half* xs = X;
  if constexpr (XS) {
    __half* xsm = reinterpret_cast<__half*>(dsmem);
    const int vec_per_row = d_in >> 3;  // 16-byte vectors per row
    for (int i = threadIdx.x; i < M * vec_per_row; i += blockDim.x) {
      const int r = i / vec_per_row, v = i - r * vec_per_row;
      *reinterpret_cast<uint4*>(xsm + (size_t)r * xstride + v * 8) =
          ld_nc_v4(X + (size_t)r * d_in + v * 8);
    }
    __syncthreads();
    xs = xsm;
  }
  const bool xrow = g < M;
  const __half* xr = xs + (size_t)g * xstride;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int it0 = 0; it0 < iters; it0 += kDictDepth) {
#pragma unroll
    for (int d = 0; d < kDictDepth; ++d) {
      const int it = it0 + d;
      if (it < iters) {
        const int u = p + it * P;
        uint32_t xw[16];
        if (xrow && u < n_units) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = XS ? *reinterpret_cast<const uint4*>(xr + (size_t)u * 32 + q * 8)
                               : ld_nc_v4(xr + (size_t)u * 32 + q * 8);
            xw[4 * q] = v.x;
            xw[4 * q + 1] = v.y;
            xw[4 * q + 2] = v.z;
            xw[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) xw[q] = 0u;
        }
        dict_unit_mma(acc, ring[d], xw);
        const int un = p + (it + kDictDepth) * P;
        load_unit(ring[d], c, s, un, (it + kDictDepth) < iters && un < n_units);
      }
    }
  }
  // acc[0], acc[1] = token g, atoms 2*tig, 2*tig+1 (acc[2], acc[3] are the zero rows g+8)
  red[warp][g][2 * tig] = acc[0][0] + acc[1][0];
  red[warp][g][2 * tig + 1] = acc[0][1] + acc[1][1];
  __syncthreads();
  if (threadIdx.x < 8 * kDictAtoms) {
    const int n = threadIdx.x / kDictAtoms, a = threadIdx.x % kDictAtoms;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kDictWarps; ++w) sum += red[w][n][a];
    if (n < mp) Z[(size_t)(tile * kDictAtoms + a) * mp + n] = sum * s_D;
  }
}

// =================================================================================
// Stage 2: coefficients
// =================================================================================
constexpr int kCoeffThreads = 512;
constexpr int kChunkEntries = 16384;
constexpr int kSegBytes = 8192;
// stage layout (bytes): idx | codes | scales | seg_start
constexpr int kStIdx = 0;
constexpr int kStCodes = kStIdx + kChunkEntries;
constexpr int kStScales = kStCodes + kChunkEntries / 2 + 16;
constexpr int kStSeg = kStScales + kChunkEntries / 16 + 32;
constexpr int kStageBytes = kStSeg + kSegBytes + 32;

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

// Segment bookkeeping: s(q) = max{s : ss[s] <= q}; `nb` = ss[s+1] (INT_MAX past the last).
__device__ __forceinline__ void advance_segment(int q, int& s, int& nb, const uint16_t* ss, int nseg) {
  while (q >= nb) {
    ++s;
    nb = (s + 1 < nseg) ? (int)ss[s + 1] : INT_MAX;
  }
}

// Sum of one 16-entry block (entries q0 .. q0+15 of a column, segment state
// valid for q0): returns blk[m] = sum_e Z[m][atom_e] * E2M1(code_e), unscaled.
// With at most one segment boundary inside the block, entry i uses segment s
// for i < t and s+1 from t on (a select); otherwise entries advance one by one.
template <int MP>
__device__ __forceinline__ void block_sum(float blk[MP], const float* zs, uint4 iv, uint2 cv, int q0, int s,
                                          int nb, const uint16_t* ss, int nseg) {
  const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
  const uint32_t cw[2] = {cv.x, cv.y};
  float a0[MP], a1[MP];  // two independent accumulation chains (even / odd entries)
#pragma unroll
  for (int m = 0; m < MP; ++m) a0[m] = a1[m] = 0.f;
  const int nb2 = (s + 2 < nseg) ? (int)ss[s + 2] : INT_MAX;
  if (q0 + 15 < nb2) {
    const int t = min(nb - q0, 16);
    const float* z0 = zs + (size_t)(s << 8) * MP;
    const float* z1 = z0 + 256 * MP;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t f[4];
      e2m1x8_to_f16x2x4(cw[j], f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[i]));
        const int e0 = 8 * j + 2 * i, e1 = e0 + 1;
        const uint32_t b0 = (iw[e0 >> 2] >> ((e0 & 3) * 8)) & 0xFFu;
        const uint32_t b1 = (iw[e1 >> 2] >> ((e1 & 3) * 8)) & 0xFFu;
        fma_z<MP>(a0, (e0 >= t ? z1 : z0) + b0 * MP, v.x);
        fma_z<MP>(a1, (e1 >= t ? z1 : z0) + b1 * MP, v.y);
      }
    }
  } else {
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
          advance_segment(q0 + ent, s, nb, ss, nseg);
          const uint32_t a = ((uint32_t)s << 8) + ((iw[ent >> 2] >> ((ent & 3) * 8)) & 0xFFu);
          fma_z<MP>(h ? a1 : a0, zs + (size_t)a * MP, h ? v.y : v.x);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) blk[m] = a0[m] + a1[m];
}

struct StageRanges {
  uint32_t codes_a0, scales_a0, seg_a0;  // 16-byte aligned source offsets
  uint32_t idx_n, codes_n, scales_n, seg_n;
};

__device__ __forceinline__ StageRanges stage_ranges(const uint4 ch, int nseg) {
  // ch = {o_b, o_e, e_b, e_e}
  StageRanges r;
  r.idx_n = ch.w - ch.z;
  r.codes_a0 = (ch.z >> 1) & ~15u;
  r.codes_n = (((ch.w >> 1) + 15u) & ~15u) - r.codes_a0;
  r.scales_a0 = (ch.z >> 4) & ~15u;
  r.scales_n = (((ch.w >> 4) + 15u) & ~15u) - r.scales_a0;
  const uint32_t sb = 2u * ch.x * (uint32_t)nseg, se = 2u * ch.y * (uint32_t)nseg;
  r.seg_a0 = sb & ~15u;
  r.seg_n = ((se + 15u) & ~15u) - r.seg_a0;
  return r;
}

__device__ __forceinline__ void issue_chunk(unsigned char* st, uint64_t* bar, const uint4 ch, int nseg,
                                           const uint8_t* idx, const uint8_t* codes, const uint8_t* scales,
                                           const uint16_t* seg_start) {
  const StageRanges r = stage_ranges(ch, nseg);
  mbar_arrive_expect_tx(bar, r.idx_n + r.codes_n + r.scales_n + r.seg_n);
  if (r.idx_n) bulk_g2s(st + kStIdx, idx + ch.z, r.idx_n, bar);
  if (r.codes_n) bulk_g2s(st + kStCodes, codes + r.codes_a0, r.codes_n, bar);
  if (r.scales_n) bulk_g2s(st + kStScales, scales + r.scales_a0, r.scales_n, bar);
  if (r.seg_n)
    bulk_g2s(st + kStSeg, reinterpret_cast<const uint8_t*>(seg_start) + r.seg_a0, r.seg_n, bar);
}

template <int MP>
__global__ void __launch_bounds__(kCoeffThreads, 2)
k_coeff_decode(const uint4* __restrict__ chunks, const int* __restrict__ cta_ptr,
               const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
               const uint8_t* __restrict__ idx, const uint16_t* __restrict__ seg_start, int nseg,
               float s_C, int k, int d_out, const float* __restrict__ Z, int M, __half* __restrict__ Y) {
  extern __shared__ __align__(128) unsigned char csmem[];
  float* zs = reinterpret_cast<float*>(csmem);                      // [k][MP]
  float* part = zs + (size_t)k * MP;                                 // [kChunkEntries/16][MP]
  unsigned char* stage0 = reinterpret_cast<unsigned char*>(part + (kChunkEntries / 16) * MP);
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage0 + 2 * kStageBytes);

  const int c0 = cta_ptr[blockIdx.x], c1 = cta_ptr[blockIdx.x + 1];
  const int nch = c1 - c0;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 && i < nch; ++i)
      issue_chunk(stage0 + i * kStageBytes, &bars[i], chunks[c0 + i], nseg, idx, codes, scales, seg_start);
  }
  trigger_dependents();
  grid_dependency_wait();  // Z comes from the dictionary stage

  for (int i = threadIdx.x * 4; i < k * MP; i += kCoeffThreads * 4)
    *reinterpret_cast<float4*>(zs + i) = *reinterpret_cast<const float4*>(Z + i);
  __syncthreads();

  for (int ci = 0; ci < nch; ++ci) {
    const int sti = ci & 1;
    unsigned char* st = stage0 + sti * kStageBytes;
    const uint4 ch = chunks[c0 + ci];
    if (!mbar_wait_bounded(&bars[sti], (ci >> 1) & 1)) break;  // error recorded; leave
    const StageRanges r = stage_ranges(ch, nseg);
    const int ncols = (int)(ch.y - ch.x);
    const int P = ncols ? (int)((ch.w - ch.z) / (uint32_t)ncols) : 0;
    const int nbc = P >> 4;
    const int nblk = ncols * nbc;
    const uint8_t* idx_s = st + kStIdx;
    const uint8_t* codes_s = st + kStCodes + ((ch.z >> 1) - r.codes_a0);
    const uint8_t* scales_s = st + kStScales + ((ch.z >> 4) - r.scales_a0);
    const uint16_t* seg_s = reinterpret_cast<const uint16_t*>(st + kStSeg + (2u * ch.x * nseg - r.seg_a0));

    // phase A: every thread sums a contiguous run of blocks (one division per
    // chunk; column and segment state advance incrementally)
    if (nblk) {
      const int R = (nblk + kCoeffThreads - 1) / kCoeffThreads;
      const int b0 = threadIdx.x * R, b1 = min(nblk, b0 + R);
      if (b0 < b1) {
        int col = b0 / nbc;
        int jb = b0 - col * nbc;
        const uint16_t* ss = seg_s + (size_t)col * nseg;
        int sgi = 0;
        for (int j = 1; j < nseg; ++j) sgi += ((int)ss[j] <= (jb << 4));
        int nb = (sgi + 1 < nseg) ? (int)ss[sgi + 1] : INT_MAX;
        uint4 iv = *reinterpret_cast<const uint4*>(idx_s + 16 * b0);
        uint2 cv = *reinterpret_cast<const uint2*>(codes_s + 8 * b0);
        uint32_t scb = scales_s[b0];
        for (int b = b0; b < b1; ++b) {
          // prefetch the next block of the run
          uint4 iv_n = iv;
          uint2 cv_n = cv;
          uint32_t sc_n = scb;
          if (b + 1 < b1) {
            iv_n = *reinterpret_cast<const uint4*>(idx_s + 16 * (b + 1));
            cv_n = *reinterpret_cast<const uint2*>(codes_s + 8 * (b + 1));
            sc_n = scales_s[b + 1];
          }
          const int q0 = jb << 4;
          float blk[MP];
          block_sum<MP>(blk, zs, iv, cv, q0, sgi, nb, ss, nseg);
          const float sc = e4m3_to_f32(scb);
#pragma unroll
          for (int m = 0; m < MP; ++m) part[b * MP + m] = blk[m] * sc;
          if (++jb == nbc) {  // next column
            jb = 0;
            ss += nseg;
            sgi = 0;
            nb = nseg > 1 ? (int)ss[1] : INT_MAX;
            advance_segment(0, sgi, nb, ss, nseg);
          } else {
            advance_segment(jb << 4, sgi, nb, ss, nseg);
          }
          iv = iv_n;
          cv = cv_n;
          scb = sc_n;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && ci + 2 < nch)
      issue_chunk(st, &bars[sti], chunks[c0 + ci + 2], nseg, idx, codes, scales, seg_start);
    // phase B: one warp per column sums its block partials in a fixed order
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int col = warp; col < ncols; col += kCoeffThreads / 32) {
      float acc[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] = 0.f;
      for (int j = lane; j < nbc; j += 32) {
#pragma unroll
        for (int m = 0; m < MP; ++m) acc[m] += part[(col * nbc + j) * MP + m];
      }
#pragma unroll
      for (int m = 0; m < MP; ++m) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
      }
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < M) Y[(size_t)m * d_out + ch.x + col] = __float2half_rn(acc[m] * s_C);
      }
    }
    __syncthreads();
  }
}

// Fallback for layers whose columns do not fit a chunk (padded column length >
// 16384 entries): lanes read blocks straight from global memory.
template <int MP>
__global__ void __launch_bounds__(256)
k_coeff_decode_direct(const uint32_t* __restrict__ col_ptr, const uint8_t* __restrict__ codes,
                      const uint8_t* __restrict__ scales, const uint8_t* __restrict__ idx,
                      const uint16_t* __restrict__ seg_start, int nseg, float s_C, int k, int d_out,
                      const float* __restrict__ Z, int M, __half* __restrict__ Y) {
  extern __shared__ __align__(16) float zsd[];  // [k + 256][MP]; the tail is zero
  trigger_dependents();
  grid_dependency_wait();
  for (int i = threadIdx.x * 4; i < k * MP; i += blockDim.x * 4)
    *reinterpret_cast<float4*>(zsd + i) = *reinterpret_cast<const float4*>(Z + i);
  // zero tail: an index byte in the last 256-atom segment never reads past the table
  for (int i = k * MP + threadIdx.x; i < (k + 256) * MP; i += blockDim.x) zsd[i] = 0.f;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * 8 + warp;
  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.f;
  if (o < d_out) {
    const uint32_t cb = col_ptr[o], ce = col_ptr[o + 1];
    const int nblk = (int)((ce - cb) >> 4);
    const uint16_t* ss = seg_start + (size_t)o * nseg;
    int s = 0, nb = nseg > 1 ? (int)ss[1] : INT_MAX;
    for (int b = lane; b < nblk; b += 32) {
      const int q0 = b << 4;
      const size_t e = cb + (size_t)q0;
      advance_segment(q0, s, nb, ss, nseg);
      float blk[MP];
      block_sum<MP>(blk, zsd, ld_stream_v4(idx + e), ld_stream_v2(codes + (e >> 1)), q0, s, nb, ss, nseg);
      const float sc = e4m3_to_f32(ld_stream_u8(scales + (e >> 4)));
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] = fmaf(blk[m], sc, acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
  }
  if (o < d_out && lane == 0) {
#pragma unroll
    for (int m = 0; m < MP; ++m)
      if (m < M) Y[(size_t)m * d_out + o] = __float2half_rn(acc[m] * s_C);
  }
}

// =================================================================================
// host side
// =================================================================================
static cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              void** args) {
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

static size_t coeff_smem(int k, int mp) {
  return (size_t)k * mp * 4 + (size_t)(kChunkEntries / 16) * mp * 4 + 2 * (size_t)kStageBytes + 16;
}

size_t coeff_decode_smem(int k, int mp) { return coeff_smem(k, mp); }

cudaError_t prepare_decode_kernels(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  // dynamic limit = opt-in limit minus the kernel's static shared memory
#define SET_SMEM(fn)                                                                                  \
  {                                                                                                   \
    cudaFuncAttributes fa;                                                                            \
    if ((e = cudaFuncGetAttributes(&fa, fn))) return e;                                               \
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,                    \
                                  optin - (int)fa.sharedSizeBytes)))                                  \
      return e;                                                                                       \
  }
  SET_SMEM(k_dict_decode<true>);
  SET_SMEM(k_dict_decode<false>);
  SET_SMEM(k_coeff_decode<1>);
  SET_SMEM(k_coeff_decode<2>);
  SET_SMEM(k_coeff_decode<4>);
  SET_SMEM(k_coeff_decode<8>);
  SET_SMEM(k_coeff_decode_direct<1>);
  SET_SMEM(k_coeff_decode_direct<2>);
  SET_SMEM(k_coeff_decode_direct<4>);
  SET_SMEM(k_coeff_decode_direct<8>);
#undef SET_SMEM
  return e;
}

cudaError_t launch_dict_decode(const dictproj_group* g, const __half* X, int M, int mp, float* Z,
                               cudaStream_t stream) {
  const uint8_t* codes = g->codes;
  const uint8_t* scales = g->scales;
  float s = g->s;
  int d_in = g->d_in;
  void* args[] = {(void*)&codes, (void*)&scales, (void*)&s, (void*)&d_in, (void*)&X,
                  (void*)&M, (void*)&mp, (void*)&Z};
  const size_t xs = (size_t)M * (d_in + 8) * sizeof(__half);
  const dim3 grid(g->k / kDictAtoms), block(kDictWarps * 32);
  if (xs <= kDictXSmemMax) return launch_pdl((const void*)k_dict_decode<true>, grid, block, xs, stream, args);
  return launch_pdl((const void*)k_dict_decode<false>, grid, block, 0, stream, args);
}

cudaError_t launch_coeff_decode(const dictproj_layer* l, const float* Z, int M, int mp, __half* Y,
                                cudaStream_t stream) {
  const uint8_t* codes = l->codes;
  const uint8_t* scales = l->scales;
  const uint8_t* idx = l->idx;
  const uint16_t* ss = l->seg_start;
  int nseg = l->nseg;
  float s = l->s;
  int k = l->k, d_out = l->d_out;
  if (l->chunks[0]) {
    const size_t smem = coeff_smem(k, mp);
    // two CTAs per SM when their shared memory (plus the 1 KB the SM reserves per CTA) fits
    const int pi = (l->chunks[1] && 2 * (smem + 1024) <= (size_t)l->smem_per_sm) ? 1 : 0;
    const uint4* chunks = reinterpret_cast<const uint4*>(l->chunks[pi]);
    const int* cta_ptr = l->cta_ptr[pi];
    void* args[] = {(void*)&chunks, (void*)&cta_ptr, (void*)&codes, (void*)&scales, (void*)&idx,
                    (void*)&ss, (void*)&nseg, (void*)&s, (void*)&k, (void*)&d_out, (void*)&Z,
                    (void*)&M, (void*)&Y};
    const dim3 grid(l->n_cta[pi]), block(kCoeffThreads);
    switch (mp) {
      case 1: return launch_pdl((const void*)k_coeff_decode<1>, grid, block, smem, stream, args);
      case 2: return launch_pdl((const void*)k_coeff_decode<2>, grid, block, smem, stream, args);
      case 4: return launch_pdl((const void*)k_coeff_decode<4>, grid, block, smem, stream, args);
      default: return launch_pdl((const void*)k_coeff_decode<8>, grid, block, smem, stream, args);
    }
  }
  const uint32_t* col_ptr = l->col_ptr;
  void* args[] = {(void*)&col_ptr, (void*)&codes, (void*)&scales, (void*)&idx, (void*)&ss,
                  (void*)&nseg, (void*)&s, (void*)&k, (void*)&d_out, (void*)&Z, (void*)&M, (void*)&Y};
  const dim3 grid((d_out + 7) / 8), block(256);
  const size_t smem = (size_t)(k + 256) * mp * sizeof(float);
  switch (mp) {
    case 1: return launch_pdl((const void*)k_coeff_decode_direct<1>, grid, block, smem, stream, args);
    case 2: return launch_pdl((const void*)k_coeff_decode_direct<2>, grid, block, smem, stream, args);
    case 4: return launch_pdl((const void*)k_coeff_decode_direct<4>, grid, block, smem, stream, args);
    default: return launch_pdl((const void*)k_coeff_decode_direct<8>, grid, block, smem, stream, args);
  }
}

// Chunk plan for k_coeff_decode: CTA c owns the columns whose first entry falls in
// [c*T/G, (c+1)*T/G); its run is cut into chunks of equal padded column length,
// at most kChunkEntries entries and at most kSegBytes of seg_start rows.
// Returns false if some column is longer than a chunk (use the direct kernel).
bool plan_coeff_chunks(const uint32_t* pcol_ptr, int d_out, int nseg, int G, std::vector<uint32_t>& chunks,
                       std::vector<int>& cta_ptr) {
  chunks.clear();
  cta_ptr.assign(G + 1, 0);
  const uint64_t T = pcol_ptr[d_out];
  const int max_cols = std::max(1, std::min(kChunkEntries, kSegBytes / (2 * nseg)));
  for (int o = 0; o < d_out; ++o)
    if (pcol_ptr[o + 1] - pcol_ptr[o] > (uint32_t)kChunkEntries) return false;
  int o = 0;
  for (int c = 0; c < G; ++c) {
    cta_ptr[c] = (int)(chunks.size() / 4);
    const uint64_t hi = (c + 1 == G) ? UINT64_MAX : (T * (uint64_t)(c + 1)) / (uint64_t)G;
    while (o < d_out && (c + 1 == G || (uint64_t)pcol_ptr[o] < hi)) {
      const uint32_t P = pcol_ptr[o + 1] - pcol_ptr[o];
      int o2 = o + 1;
      while (o2 < d_out && (c + 1 == G || (uint64_t)pcol_ptr[o2] < hi) &&
             pcol_ptr[o2 + 1] - pcol_ptr[o2] == P && (uint64_t)(o2 + 1 - o) * P <= (uint64_t)kChunkEntries &&
             o2 + 1 - o <= max_cols)
        ++o2;
      chunks.push_back((uint32_t)o);
      chunks.push_back((uint32_t)o2);
      chunks.push_back(pcol_ptr[o]);
      chunks.push_back(pcol_ptr[o2]);
      o = o2;
    }
  }
  cta_ptr[G] = (int)(chunks.size() / 4);
  return true;
}

cudaError_t take_decode_error(unsigned int* out) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_dictproj_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_dictproj_error, &zero, sizeof(unsigned int));
}

}  // namespace dictproj
