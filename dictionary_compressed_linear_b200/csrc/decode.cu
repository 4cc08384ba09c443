// Decode path (M <= 8 tokens): the two stages of Eq. (1) of the DictLLM
// technical review, Z = X D_g then Y = Z C_l, as two kernels chained with
// programmatic dependent launch. Both issue the reads of their packed weights
// before waiting on the previous kernel (nothing writes weights after upload),
// so weight traffic overlaps the tail of the preceding work on the stream.
//
// Stage 1, dictionary (HBM-bound GEMV over packed NVFP4 D_g), k_dict_decode.
//   The grid is (k/16 atom tiles) x (d_in slices); each warp owns whole units of
//   16 atoms x 128 d_in elements, J of them, with one J for a whole batched call
//   chosen by a fitted wave cost (dict_plan_batch). A thread streams the 16-byte
//   code words of two atoms through a register ring (raw weights are loaded
//   before the dependency wait; a bulk L2 prefetch covers the rest of the CTA's
//   slice), converts E2M1
//   pairs to f16x2 with the hardware cvt, multiplies by the E4M3 block scale in
//   fp16 (an E2M1 x E4M3 product is exact in fp16), and issues mma.sync m16n8k16
//   with the atoms as the 16 rows of A and the tokens as the 8 columns of B, fp32
//   accumulate. Warp partials are reduced in shared memory in a fixed order and
//   each slice writes s_D * partial to Zpart[slice][k][mp].
//
// Stage 2, coefficients (sparse gather over column-compressed NVFP4 C_l),
// k_coeff_gather.
//   One CTA per SM (1024 threads) owns a contiguous run of columns, one warp per
//   column; a batched call hands its CTAs to the projection that would finish
//   last (gather_batch_shares). Z = the sum of the dictionary stage's slices
//   (fixed order) is staged in shared memory as an fp16 table with a zero tail.
//   A column's entries (index bytes, codes, scales, seg_start) are loaded
//   straight from global memory into registers, the first column before the
//   dependency wait and each next one while the current one is summed: lane l
//   takes the 8-entry half-blocks 32i + l of the column (atom = 256*segment +
//   idx; the segment of each half-block comes from one ballot and one OR-reduced
//   mask of the 8-rounded segment starts per 256-entry window, and a column with
//   two starts inside one half-block walks its entries instead), multiplies fp16
//   Z by the fp16 E2M1 value with fma.rn.f32.f16, scales each half-block by its
//   E4M3 block scale, and the warp reduces with shuffles in a fixed order, so
//   results are bit-reproducible. Y = s_C * sum in fp16. Columns longer than 1280
//   stored entries, or k above 8192 atoms, go to k_coeff_decode_direct (one warp
//   per column, lanes over 16-entry blocks, any length; fp32 Z).

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
constexpr int kDictWarps = 8;     // warps per CTA; each owns whole 128-element units
constexpr int kDictTile = 16;     // atoms per CTA = MMA M

// A unit is 16 atoms x 128 d_in elements: thread (g, t) of a warp holds atoms g
// and g+8 of the tile and elements [128u + 32t, 128u + 32t + 32).
// By-value launch descriptors for batches of independent projections.
constexpr int kMaxBatch = 4;
struct DictProj {
  const uint8_t* codes;
  const uint8_t* scales;
  const __half* X;
  float* Zpart;
  float s;
  int d_in, k, J, tiles, block_begin;
};
struct DictBatch {
  DictProj p[kMaxBatch];
  int n, M, mp;
};
struct CoeffProj {
  const uint32_t* col_ptr;
  const uint8_t* codes;
  const uint8_t* scales;
  const uint8_t* idx;
  const uint16_t* seg_start;
  const float* Zpart;
  __half* Y;
  float s;
  int nseg, k, d_out, nslices, cols_per_cta, block_begin;
};
struct CoeffBatch {
  CoeffProj p[kMaxBatch];
  int n, M;
};

struct DictUnit {
  uint4 wa, wb;      // 16 code bytes of atoms g and g+8 (32 elements each)
  uint32_t sa, sb;   // their two E4M3 block scales (2 bytes each)
};

__device__ __forceinline__ void load_unit(DictUnit& u, const uint8_t* c0, const uint8_t* c1, const uint8_t* s0,
                                          const uint8_t* s1, size_t off_c, size_t off_s, bool ok) {
  if (ok) {
    u.wa = ld_stream_v4(c0 + off_c);
    u.wb = ld_stream_v4(c1 + off_c);
    u.sa = ld_stream_u16(s0 + off_s);
    u.sb = ld_stream_u16(s1 + off_s);
  } else {
    u.wa = make_uint4(0, 0, 0, 0);
    u.wb = u.wa;
    u.sa = u.sb = 0;
  }
}

// One unit: 8 MMAs m16n8k16 with the atoms as the 16 rows of A (swap-AB) and the
// tokens as the 8 columns of B; 4 elements per thread per MMA.
// A: a0:a1 <- atom g, elements 8q+4h+{0,1}; a2:a3 <- atom g+8, same; a4:a5 / a6:a7 <- +{2,3}.
// B: b0:b1 <- X[token g][same elements +{0,1}], b2:b3 <- +{2,3}.
template <bool XS>
__device__ __forceinline__ void dict_unit_mma(float acc[2][4], const DictUnit& u, const __half* px, bool xon) {
  const uint32_t ha = e4m3x2_to_f16x2(u.sa), hb = e4m3x2_to_f16x2(u.sb);
  const uint32_t wa[4] = {u.wa.x, u.wa.y, u.wa.z, u.wa.w};
  const uint32_t wb[4] = {u.wb.x, u.wb.y, u.wb.z, u.wb.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t fa[4], fb[4];
    e2m1x8_to_f16x2x4(wa[q], fa);
    e2m1x8_to_f16x2x4(wb[q], fb);
    const uint32_t sa = q < 2 ? dup_lo(ha) : dup_hi(ha);
    const uint32_t sb = q < 2 ? dup_lo(hb) : dup_hi(hb);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      fa[i] = hmul2_u32(fa[i], sa);  // E2M1 x E4M3 is exact in fp16
      fb[i] = hmul2_u32(fb[i], sb);
    }
    uint4 xv = make_uint4(0, 0, 0, 0);  // X elements 8q .. 8q+7 of this thread's range
    if (xon) xv = XS ? *reinterpret_cast<const uint4*>(px + 8 * q) : ld_nc_v4(px + 8 * q);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a[4] = {fa[2 * h], fb[2 * h], fa[2 * h + 1], fb[2 * h + 1]};
      const uint32_t b[2] = {xw[2 * h], xw[2 * h + 1]};
      mma_16816(acc[h], a, b);  // two independent accumulation chains
    }
  }
}

// Zpart[slice][atom][mp] = s_D * sum over the slice's units of X[m][i] * D[i][atom].
// One launch serves up to kMaxBatch independent projections; projection i owns
// blocks [block_begin, block_begin + tiles * slices) of the 1-D grid, block
// (tile, slice) = (local % tiles, local / tiles); slice y covers units
// [y*8*J, (y+1)*8*J).
// RING = register prefetch depth in units (1, 2 or 4; at most J is useful).
// XS: X rows of the slice are staged in shared memory (stride xlen + 8 halves).
template <int RING, bool XS>
__global__ void __launch_bounds__(kDictWarps * 32, 4)  // at most 64 registers
k_dict_decode(const __grid_constant__ DictBatch batch) {
  extern __shared__ __align__(16) unsigned char dsmem[];
  __shared__ float red[kDictWarps][kDictTile][8];
  // projection of this CTA; its blocks are [block_begin, block_begin + tiles * slices)
  int pi = 0;
  while (pi + 1 < batch.n && (int)blockIdx.x >= batch.p[pi + 1].block_begin) ++pi;
  const DictProj& pr = batch.p[pi];
  const uint8_t* __restrict__ codes = pr.codes;
  const uint8_t* __restrict__ scales = pr.scales;
  const float s_D = pr.s;
  const int d_in = pr.d_in, k = pr.k, J = pr.J;
  const __half* __restrict__ X = pr.X;
  float* __restrict__ Zpart = pr.Zpart;
  const int M = batch.M, mp = batch.mp;
  const int local = (int)blockIdx.x - pr.block_begin;
  const int tile = local % pr.tiles, slice = local / pr.tiles;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const size_t crow = (size_t)(d_in >> 1), srow = (size_t)(d_in >> 4);
  const uint8_t* c0 = codes + (size_t)(tile * kDictTile + g) * crow;
  const uint8_t* c1 = c0 + 8 * crow;
  const uint8_t* s0 = scales + (size_t)(tile * kDictTile + g) * srow;
  const uint8_t* s1 = s0 + 8 * srow;
  const int u_begin = slice * kDictWarps * J;
  const int e_begin = u_begin * 128;
  const int e_end = min(d_in, (u_begin + kDictWarps * J) * 128);
  // element range of this thread in unit u: [128u + 32t, +32); valid iff it ends <= d_in
  auto unit_of = [&](int j) { return u_begin + warp + kDictWarps * j; };
  auto valid = [&](int u) { return 128 * u + 32 * t + 32 <= d_in; };

  if (threadIdx.x < kDictTile) {  // L2 prefetch of this CTA's slice of the 16 atom rows
    const size_t row = (size_t)(tile * kDictTile + threadIdx.x);
    prefetch_l2_range(codes, row * crow + e_begin / 2, row * crow + e_end / 2);
    prefetch_l2_range(scales, row * srow + e_begin / 16, row * srow + e_end / 16);
  }
  DictUnit ring[RING];
#pragma unroll
  for (int d = 0; d < RING; ++d) {
    const int u = unit_of(d);
    load_unit(ring[d], c0, c1, s0, s1, (size_t)u * 64 + 16 * t, (size_t)u * 8 + 2 * t, d < J && valid(u));
  }
  trigger_dependents();
  grid_dependency_wait();  // X and the Z scratch belong to earlier work on the stream

  const int xlen = e_end - e_begin;
  const int xstride = XS ? xlen + 8 : d_in;
  const __half* xr;
  if constexpr (XS) {  // stage X[0:M][slice] once; one L2 round trip for the whole CTA
    __half* xsm = reinterpret_cast<__half*>(dsmem);
    const int vpr = xlen >> 3;  // 16-byte vectors per row
    for (int i = threadIdx.x; i < M * vpr; i += blockDim.x) {
      const int r = i / vpr, v = i - r * vpr;
      *reinterpret_cast<uint4*>(xsm + (size_t)r * xstride + 8 * v) =
          ld_nc_v4(X + (size_t)r * d_in + e_begin + 8 * v);
    }
    __syncthreads();
    xr = xsm + (size_t)g * xstride - e_begin;  // index with absolute element numbers
  } else {
    xr = X + (size_t)g * d_in;
  }
  const bool xrow = g < M;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int j0 = 0; j0 < J; j0 += RING) {
#pragma unroll
    for (int d = 0; d < RING; ++d) {
      const int j = j0 + d;
      if (j < J) {
        const int u = unit_of(j);
        dict_unit_mma<XS>(acc, ring[d], xr + (size_t)u * 128 + 32 * t, xrow && valid(u));
        const int un = unit_of(j + RING);
        load_unit(ring[d], c0, c1, s0, s1, (size_t)un * 64 + 16 * t, (size_t)un * 8 + 2 * t,
                  j + RING < J && valid(un));
      }
    }
  }
  // c0:c1 = atom g, tokens 2t, 2t+1; c2:c3 = atom g+8, tokens 2t, 2t+1
  red[warp][g][2 * t] = acc[0][0] + acc[1][0];
  red[warp][g][2 * t + 1] = acc[0][1] + acc[1][1];
  red[warp][g + 8][2 * t] = acc[0][2] + acc[1][2];
  red[warp][g + 8][2 * t + 1] = acc[0][3] + acc[1][3];
  __syncthreads();
  if (threadIdx.x < kDictTile * 8) {
    const int a = threadIdx.x >> 3, n = threadIdx.x & 7;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kDictWarps; ++w) sum += red[w][a][n];
    if (n < mp) Zpart[((size_t)slice * k + tile * kDictTile + a) * mp + n] = sum * s_D;
  }
}

// =================================================================================
// Stage 2: coefficients
// =================================================================================
// seg_start row reader (global row).
struct SegGlobal {
  const uint16_t* p;
  __device__ __forceinline__ int operator()(int j) const { return (int)p[j]; }
};

// Segment bookkeeping: s(q) = max{s : ss[s] <= q}; `nb` = ss[s+1] (INT_MAX past the last).
template <class SS>
__device__ __forceinline__ void advance_segment(int q, int& s, int& nb, const SS& ss, int nseg) {
  while (q >= nb) {
    ++s;
    nb = (s + 1 < nseg) ? ss(s + 1) : INT_MAX;
  }
}

// Sum of NE consecutive entries (q0 .. q0+NE-1 of a column; segment state valid
// for q0) given their index bytes `iw` and codes `cw`; unscaled. Z is read from
// shared memory at zaddr (32-bit addresses throughout).
// With at most one segment boundary inside, entry i uses segment s for i < t and
// s+1 from t on (a select); otherwise the entries advance one by one.
template <int MP, int NE, class SS>
__device__ __forceinline__ void entries_sum(float blk[MP], uint32_t zaddr, const uint32_t* iw, const uint32_t* cw,
                                            int q0, int s, int nb, int nb2, const SS& ss, int nseg) {
  // nb, nb2: the first two segment starts after q0 (INT_MAX if none)
  constexpr uint32_t kRow = MP * 4;  // bytes per atom row of Z
  float a0[MP], a1[MP];              // two independent accumulation chains (even / odd entries)
#pragma unroll
  for (int m = 0; m < MP; ++m) a0[m] = a1[m] = 0.f;
  if (q0 + NE - 1 < nb2) {
    const int t = min(nb - q0, NE);
    const uint32_t z0 = zaddr + ((uint32_t)s << 8) * kRow;
    const uint32_t z1 = z0 + 256u * kRow;
#pragma unroll
    for (int j = 0; j < NE / 8; ++j) {
      uint32_t f[4];
      e2m1x8_to_f16x2x4(cw[j], f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[i]));
        const int e0 = 8 * j + 2 * i, e1 = e0 + 1;
        const uint32_t b0 = __byte_perm(iw[e0 >> 2], 0u, 0x4440u | (uint32_t)(e0 & 3));
        const uint32_t b1 = __byte_perm(iw[e1 >> 2], 0u, 0x4440u | (uint32_t)(e1 & 3));
        fma_z<MP>(a0, (e0 >= t ? z1 : z0) + b0 * kRow, v.x);
        fma_z<MP>(a1, (e1 >= t ? z1 : z0) + b1 * kRow, v.y);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < NE / 8; ++j) {
      uint32_t f[4];
      e2m1x8_to_f16x2x4(cw[j], f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[i]));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ent = 8 * j + 2 * i + h;
          advance_segment(q0 + ent, s, nb, ss, nseg);
          const uint32_t b = __byte_perm(iw[ent >> 2], 0u, 0x4440u | (uint32_t)(ent & 3));
          fma_z<MP>(h ? a1 : a0, zaddr + (((uint32_t)s << 8) + b) * kRow, h ? v.y : v.x);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) blk[m] = a0[m] + a1[m];
}

// Stage Z (sum of the dictionary stage's slices, fixed order) into shared memory.
// The slices' loads are issued four at a time before any of them is summed, so
// the staging costs one L2 round trip per four slices, not one per slice; the
// sum keeps the slice order (bit-identical to a plain loop).
template <int MP>
__device__ __forceinline__ void stage_z(float* zs, const float* __restrict__ Zpart, int nslices, int k, int nthr) {
  const int n = k * MP;
  for (int i = threadIdx.x * 4; i < n; i += nthr * 4) {
    float4 a = ld_cg_v4f(Zpart + i);
    for (int s0 = 1; s0 < nslices; s0 += 4) {
      float4 b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (s0 + j < nslices) b[j] = ld_cg_v4f(Zpart + (size_t)(s0 + j) * n + i);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (s0 + j < nslices) {
          a.x += b[j].x;
          a.y += b[j].y;
          a.z += b[j].z;
          a.w += b[j].w;
        }
    }
    *reinterpret_cast<float4*>(zs + i) = a;
  }
}

// stage_z, rounded to an fp16 table (the gather kernel's Z).
template <int MP>
__device__ __forceinline__ void stage_zh(__half* zs, const float* __restrict__ Zpart, int nslices, int k, int nthr) {
  const int n = k * MP;
  for (int i = threadIdx.x * 4; i < n; i += nthr * 4) {
    float4 a = ld_cg_v4f(Zpart + i);
    for (int s0 = 1; s0 < nslices; s0 += 4) {
      float4 b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (s0 + j < nslices) b[j] = ld_cg_v4f(Zpart + (size_t)(s0 + j) * n + i);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (s0 + j < nslices) {
          a.x += b[j].x;
          a.y += b[j].y;
          a.z += b[j].z;
          a.w += b[j].w;
        }
    }
    __half2* d = reinterpret_cast<__half2*>(zs + i);
    d[0] = __floats2half2_rn(a.x, a.y);
    d[1] = __floats2half2_rn(a.z, a.w);
  }
}

// Gather kernel (k_coeff_gather) for columns of at most kRmax*256 entries and k
// of at most 32*256 atoms (nseg <= 32): one warp per column, lanes interleaved
// over 8-entry half-blocks (coalesced, conflict-free loads straight from
// global/L2), the column's loads double-buffered in registers across the warp's
// columns, and the column's seg_start row held one value per lane.
constexpr int kRmax = 5;         // steps of 32 half-blocks held per column
static_assert(kRmax <= 8, "one scale byte per step in a 64-bit word");
constexpr int kGatherWarps = 32;

struct ColData {
  uint2 iv[kRmax];      // 8 index bytes per step
  uint32_t cv[kRmax];   // 8 codes (4 bytes) per step
  uint64_t sc;          // E4M3 scale byte of each step, packed 8 bits apiece (kRmax <= 8)
  int ssv;              // seg_start[lane] of the column (lane < nseg), else INT_MAX
};

// The column's loads: lane L takes half-blocks L, L + 32, ... through per-lane
// base pointers, so every step is one load per stream at a constant offset.
__device__ __forceinline__ void load_col(ColData& d, int o, int d_out, const uint32_t* __restrict__ col_ptr,
                                         const uint8_t* __restrict__ idx, const uint8_t* __restrict__ codes,
                                         const uint8_t* __restrict__ scales, const uint16_t* __restrict__ seg_start,
                                         int nseg, int lane, int& nhb) {
  nhb = 0;
  d.sc = 0;
  d.ssv = INT_MAX;
#pragma unroll
  for (int i = 0; i < kRmax; ++i) {
    d.iv[i] = make_uint2(0, 0);
    d.cv[i] = 0;
  }
  if (o >= d_out) return;
  const uint32_t cb = col_ptr[o];
  nhb = (int)((col_ptr[o + 1] - cb) >> 3);
  if (lane < nseg) d.ssv = (int)seg_start[(size_t)o * nseg + lane];
  const uint8_t* pi = idx + cb + 8 * lane;
  const uint8_t* pc = codes + (cb >> 1) + 4 * lane;
  const uint8_t* ps = scales + (cb >> 4) + (lane >> 1);
#pragma unroll
  for (int i = 0; i < kRmax; ++i) {
    if (32 * i + lane < nhb) {
      d.iv[i] = ld_stream_v2(pi + 256 * i);
      d.cv[i] = *reinterpret_cast<const uint32_t*>(pc + 128 * i);
      d.sc |= (uint64_t)ld_stream_u8(ps + 16 * i) << (8 * i);
    }
  }
}

// One column of the gather: Y[m][o] = s_C * sum over the column's stored
// entries of Z[m][atom] * value (d holds the column's entries, loaded earlier).
template <int MP>
__device__ __forceinline__ void gather_column(const ColData& d, int o, int nhb, uint32_t zs_a, int nseg,
                                              const uint16_t* __restrict__ seg_start, int lane, int M, int d_out,
                                              float s_C, __half* __restrict__ Y) {
  constexpr uint32_t kRowH = MP * 2;  // bytes per atom row of the fp16 Z table
  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.f;
  // Lane j (1 <= j < nseg) holds the start of segment j and c_j, that start
  // rounded up to a multiple of 8. The segment of the half-block starting at q0
  // is the number of c_j <= q0. In the window of 256 entries starting at w, c_j
  // with 0 < c_j - w < 256 counts from lane (c_j - w) / 8 on, so one OR-reduced
  // lane mask and one ballot give every lane its segment. Two starts with the
  // same c_j (two boundaries inside one half-block, or an empty segment) would
  // share a mask bit: such a column takes the walk below for every half-block.
  const bool is_bnd = lane >= 1 && lane < nseg;
  const int c = is_bnd ? ((d.ssv + 7) & ~7) : INT_MAX;
  const int c_up = __shfl_down_sync(0xffffffffu, c, 1);  // every lane takes part
  const bool dup = is_bnd && lane + 1 < nseg && c_up == c;
  const bool col_walk = __any_sync(0xffffffffu, dup);
  const uint32_t le = lane == 31 ? 0xffffffffu : ((2u << lane) - 1u);
#pragma unroll
  for (int i = 0; i < kRmax; ++i) {
    const int w = 256 * i;
    if (w >= 8 * nhb) break;
    const int t = c - w;  // a multiple of 8 (INT_MAX - w off the boundary lanes)
    const int s_lo = __popc(__ballot_sync(0xffffffffu, t <= 0));
    const uint32_t A = __reduce_or_sync(0xffffffffu, (uint32_t)(t - 1) < 255u ? (1u << ((t >> 3) & 31)) : 0u);
    const int sgi = s_lo + __popc(A & le);  // segment of q0
    const int q0 = w + 8 * lane;
    // the start of segment sgi+1 is the first boundary after q0
    const int nxt = __shfl_sync(0xffffffffu, d.ssv, min(sgi + 1, 31));
    const int t1 = sgi + 1 < nseg ? nxt : INT_MAX;
    const int t2 = col_walk ? q0 : INT_MAX;  // forces the walk
    if (32 * i + lane < nhb) {
      const uint32_t iw[2] = {d.iv[i].x, d.iv[i].y};
      float a0[MP], a1[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) a0[m] = a1[m] = 0.f;
      uint32_t f[4];
      e2m1x8_to_f16x2x4(d.cv[i], f);
      if (q0 + 7 < t2) {  // at most one boundary: entries e >= t use segment sgi+1
        const int t = min(t1 - q0, 8);
        // flag byte of each entry: 1 past the boundary; prmt then forms the
        // entry's 9-bit row (index byte + 256 x flag) with zero upper bytes
        const uint32_t fl[2] = {shl_clamped(0x01010101u, 8u * (uint32_t)t),
                                shl_clamped(0x01010101u, 8u * (uint32_t)max(t - 4, 0))};
        const uint32_t z0 = zs_a + ((uint32_t)sgi << 8) * kRowH;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t j = (uint32_t)(e & 3);
          const uint32_t row = prmt(iw[e >> 2], fl[e >> 2], j | ((4u + j) << 4) | ((12u + j) << 8) | ((12u + j) << 12));
          if (e & 1)
            fma_zh<MP, 1>(a1, z0 + row * kRowH, f[e >> 1]);
          else
            fma_zh<MP, 0>(a0, z0 + row * kRowH, f[e >> 1]);
        }
      } else {  // several boundaries inside these 8 entries: walk them (row read from memory)
        const uint16_t* ssrow = seg_start + (size_t)o * nseg;
        int sg = 0;
        for (int j = 1; j < nseg; ++j) sg += ((int)ssrow[j] <= q0);
        int nb = (sg + 1 < nseg) ? (int)ssrow[sg + 1] : INT_MAX;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          while (q0 + e >= nb) {
            ++sg;
            nb = (sg + 1 < nseg) ? (int)ssrow[sg + 1] : INT_MAX;
          }
          const uint32_t b = __byte_perm(iw[e >> 2], 0u, 0x4440u | (uint32_t)(e & 3));
          const uint32_t ad = zs_a + (((uint32_t)sg << 8) + b) * kRowH;
          if (e & 1)
            fma_zh<MP, 1>(a1, ad, f[e >> 1]);
          else
            fma_zh<MP, 0>(a0, ad, f[e >> 1]);
        }
      }
      const float sc = e4m3_to_f32_int((uint32_t)(d.sc >> (8 * i)) & 0xFFu);
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] = fmaf(a0[m] + a1[m], sc, acc[m]);
    }
  }
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

// Diagnostic: when set, each gather CTA writes the start of its column work (Z
// staged) and its end (the GPU's global timer, ns) to g_gather_times[2 * CTA]
// and [2 * CTA + 1], CTA < g_gather_ctas.
static __constant__ unsigned long long* g_gather_times;
static __constant__ int g_gather_ctas;
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

template <int MP>
__global__ void __launch_bounds__(kGatherWarps * 32, 1)  // 1024 threads, at most 64 registers
k_coeff_gather(const __grid_constant__ CoeffBatch batch) {
  extern __shared__ __align__(16) __half zsg[];  // fp16 [k + 256][MP]; the tail is zero
  unsigned long long* const tdiag = (int)blockIdx.x < g_gather_ctas ? g_gather_times : nullptr;
  int pi = 0;
  while (pi + 1 < batch.n && (int)blockIdx.x >= batch.p[pi + 1].block_begin) ++pi;
  const CoeffProj& pr = batch.p[pi];
  const uint32_t* __restrict__ col_ptr = pr.col_ptr;
  const uint8_t* __restrict__ codes = pr.codes;
  const uint8_t* __restrict__ scales = pr.scales;
  const uint8_t* __restrict__ idx = pr.idx;
  const uint16_t* __restrict__ seg_start = pr.seg_start;
  const int nseg = pr.nseg, k = pr.k, d_out = pr.d_out, nslices = pr.nslices, cols_per_cta = pr.cols_per_cta;
  const float s_C = pr.s;
  const float* __restrict__ Zpart = pr.Zpart;
  __half* __restrict__ Y = pr.Y;
  const int M = batch.M;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o_begin = ((int)blockIdx.x - pr.block_begin) * cols_per_cta;
  const int o_end = min(d_out, o_begin + cols_per_cta);
  if (threadIdx.x == 0 && o_begin < o_end) {  // bulk L2 prefetch of this CTA's columns
    const size_t e0 = col_ptr[o_begin], e1 = col_ptr[o_end];
    prefetch_l2_range(idx, e0, e1);
    prefetch_l2_range(codes, e0 >> 1, e1 >> 1);
    prefetch_l2_range(scales, e0 >> 4, e1 >> 4);
    prefetch_l2_range(seg_start, (size_t)o_begin * nseg * 2, (size_t)o_end * nseg * 2);
  }
  // Two column buffers in ping-pong: the next column's loads are in flight while
  // this one is summed, and no buffer is ever copied (a copy would wait for them).
  ColData ca, cbuf;
  int na, nb;
  int o = o_begin + warp;
  load_col(ca, o, o_end, col_ptr, idx, codes, scales, seg_start, nseg, lane, na);
  trigger_dependents();
  grid_dependency_wait();  // Z comes from the dictionary stage

  stage_zh<MP>(zsg, Zpart, nslices, k, blockDim.x);
  for (int i = k * MP + threadIdx.x; i < (k + 256) * MP; i += blockDim.x) zsg[i] = __float2half_rn(0.f);
  __syncthreads();
  const uint32_t zs_a = smem_u32(zsg);
  if (tdiag && threadIdx.x == 0) tdiag[2 * blockIdx.x] = global_ns();

  for (; o < o_end; o += 2 * kGatherWarps) {
    load_col(cbuf, o + kGatherWarps, o_end, col_ptr, idx, codes, scales, seg_start, nseg, lane, nb);
    gather_column<MP>(ca, o, na, zs_a, nseg, seg_start, lane, M, d_out, s_C, Y);
    if (o + kGatherWarps >= o_end) break;
    load_col(ca, o + 2 * kGatherWarps, o_end, col_ptr, idx, codes, scales, seg_start, nseg, lane, na);
    gather_column<MP>(cbuf, o + kGatherWarps, nb, zs_a, nseg, seg_start, lane, M, d_out, s_C, Y);
  }
  if (tdiag) {  // the same for every thread of the CTA
    __syncthreads();
    if (threadIdx.x == 0) tdiag[2 * blockIdx.x + 1] = global_ns();
  }
}

// Direct kernel, for layers the gather does not hold (a column longer than
// kRmax*256 stored entries, or more than 32 segments) and for the no-allocation
// forward: one warp per column, lanes over 16-entry blocks read straight from
// global memory, any column length.
template <int MP>
__global__ void __launch_bounds__(256)
k_coeff_decode_direct(const uint32_t* __restrict__ col_ptr, const uint8_t* __restrict__ codes,
                      const uint8_t* __restrict__ scales, const uint8_t* __restrict__ idx,
                      const uint16_t* __restrict__ seg_start, int nseg, float s_C, int k, int d_out,
                      const float* __restrict__ Zpart, int nslices, int M, __half* __restrict__ Y) {
  extern __shared__ __align__(16) float zsd[];  // [k + 256][MP]; the tail is zero
  trigger_dependents();
  grid_dependency_wait();
  stage_z<MP>(zsd, Zpart, nslices, k, blockDim.x);
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
    const SegGlobal ss{seg_start + (size_t)o * nseg};
    int s = 0, nb = nseg > 1 ? ss(1) : INT_MAX;
    const uint32_t zs_a = smem_u32(zsd);
    for (int b = lane; b < nblk; b += 32) {
      const int q0 = b << 4;
      const size_t e = cb + (size_t)q0;
      advance_segment(q0, s, nb, ss, nseg);
      const uint4 iv = ld_stream_v4(idx + e);
      const uint2 cv = ld_stream_v2(codes + (e >> 1));
      const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
      const uint32_t cw[2] = {cv.x, cv.y};
      float blk[MP];
      entries_sum<MP, 16>(blk, zs_a, iw, cw, q0, s, nb, (s + 2 < nseg) ? ss(s + 2) : INT_MAX, ss, nseg);
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

// Opt-in shared memory per block of each device, recorded by prepare_decode_kernels.
constexpr int kMaxDevices = 64;
static int g_smem_optin[kMaxDevices];

int smem_optin_of(int device) { return device >= 0 && device < kMaxDevices ? g_smem_optin[device] : 0; }

bool coeff_smem_fits(int k, int mp, int device) {
  if (device < 0 || device >= kMaxDevices) return false;
  return (size_t)(k + 256) * mp * sizeof(float) <= (size_t)g_smem_optin[device];
}

// Dictionary-stage grid: (k/16 tiles) x slices, each warp J units of 128
// elements. J is the smallest count that keeps at most two CTAs per SM and
// lets the M rows of the slice's X fit kDictXsMax bytes of shared memory;
// one_slice forces a single slice (Z written complete).
constexpr size_t kDictXsMax = 96 * 1024;

static size_t dict_xs_bytes(int xlen, int M) { return (size_t)M * (xlen + 8) * sizeof(__half); }

// Cost of a dictionary grid in rows of D streamed by one CTA: the launch takes
// ceil(CTAs / (4 x n_sm)) waves (four 256-thread CTAs fill an SM's registers),
// each as long as its longest CTA, and a CTA costs a fixed part (launch, X
// staging, the cross-warp reduction) worth kDictFixedRows rows plus its rows.
// Fitted on B200 to the LLaMA-7B shapes at M = 1 (q/k/v and gate/up batches, o
// and down alone, J = 1..8): it picks the fastest J measured for each.
constexpr long kDictFixedRows = 1700;

void dict_plan_batch(int n, const int* d_in, const int* k, int n_sm, int M, DictPlan* plans) {
  // One J for the whole batch (every CTA then streams the same 8 x J units of 16
  // atom rows, or all of a shorter d_in, so each projection's CTAs follow its
  // dictionary bytes), chosen by the cost above. Per projection, J is capped at
  // the units one slice needs and shrinks back while the slice's X rows would not
  // fit the shared-memory cap.
  int jmax = 1;
  for (int i = 0; i < n; ++i) jmax = std::max(jmax, ((d_in[i] + 127) / 128 + kDictWarps - 1) / kDictWarps);
  int best = 1;
  long best_cost = LONG_MAX;
  for (int J = 1; J <= jmax; ++J) {
    long ctas = 0, rows = 0;
    for (int i = 0; i < n; ++i) {
      const int units = (d_in[i] + 127) / 128;
      const int slices = (units + kDictWarps * J - 1) / (kDictWarps * J);
      ctas += (long)(k[i] / kDictTile) * slices;
      rows = std::max(rows, (long)std::min(d_in[i], kDictWarps * J * 128));
    }
    const long cost = (ctas + 4L * n_sm - 1) / (4L * n_sm) * (kDictFixedRows + rows);
    if (cost < best_cost) best_cost = cost, best = J;
  }
  for (int i = 0; i < n; ++i) {
    const int units = (d_in[i] + 127) / 128;
    DictPlan& p = plans[i];
    p.J = std::min(best, (units + kDictWarps - 1) / kDictWarps);
    while (p.J > 1 && dict_xs_bytes(std::min(d_in[i], kDictWarps * p.J * 128), M) > kDictXsMax) --p.J;
    p.slices = (units + kDictWarps * p.J - 1) / (kDictWarps * p.J);
  }
}

DictPlan dict_plan(int d_in, int k, int n_sm, int M, bool one_slice) {
  DictPlan p;
  if (!one_slice) {
    dict_plan_batch(1, &d_in, &k, n_sm, M, &p);
    return p;
  }
  const int units = (d_in + 127) / 128;
  p.J = (units + kDictWarps - 1) / kDictWarps;
  p.slices = 1;
  return p;
}

int dict_max_slices(int d_in, int k, int n_sm) {
  (void)k;
  (void)n_sm;
  return ((d_in + 127) / 128 + kDictWarps - 1) / kDictWarps;  // J = 1, the most any plan takes
}

cudaError_t prepare_decode_kernels(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  if (device >= 0 && device < kMaxDevices) g_smem_optin[device] = optin;
  // dynamic limit = opt-in limit minus the kernel's static shared memory
#define SET_SMEM(fn)                                                                                  \
  {                                                                                                   \
    cudaFuncAttributes fa;                                                                            \
    if ((e = cudaFuncGetAttributes(&fa, fn))) return e;                                               \
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,                    \
                                  optin - (int)fa.sharedSizeBytes)))                                  \
      return e;                                                                                       \
  }
  SET_SMEM((k_dict_decode<1, true>));
  SET_SMEM(k_coeff_gather<1>);
  SET_SMEM(k_coeff_gather<2>);
  SET_SMEM(k_coeff_gather<4>);
  SET_SMEM(k_coeff_gather<8>);
  SET_SMEM(k_coeff_decode_direct<1>);
  SET_SMEM(k_coeff_decode_direct<2>);
  SET_SMEM(k_coeff_decode_direct<4>);
  SET_SMEM(k_coeff_decode_direct<8>);
#undef SET_SMEM
  return e;
}

cudaError_t launch_dict_decode_batch(int n, const dictproj_group* const* g, const __half* const* X, int M,
                                     int mp, float* const* Zpart, const DictPlan* plans, cudaStream_t stream) {
  DictBatch b{};
  b.n = n;
  b.M = M;
  b.mp = mp;
  int blocks = 0;
  size_t xs = 0;
  for (int i = 0; i < n; ++i) {
    DictProj& p = b.p[i];
    p.codes = g[i]->codes;
    p.scales = g[i]->scales;
    p.s = g[i]->s;
    p.d_in = g[i]->d_in;
    p.k = g[i]->k;
    p.X = X[i];
    p.Zpart = Zpart[i];
    p.J = plans[i].J;
    p.tiles = g[i]->k / kDictTile;
    p.block_begin = blocks;
    blocks += p.tiles * plans[i].slices;
    xs = std::max(xs, dict_xs_bytes(std::min(p.d_in, kDictWarps * p.J * 128), M));
  }
  void* args[] = {(void*)&b};
  const dim3 grid(blocks), block(kDictWarps * 32);
  const bool use_xs = xs <= 200 * 1024;
  const size_t smem = use_xs ? xs : 0;
  // One unit in flight per warp (RING = 1): on B200 it measured as fast as two or
  // four for J = 2..8, with the CTA's slice already on its way to L2.
  return use_xs ? launch_pdl((const void*)k_dict_decode<1, true>, grid, block, smem, stream, args)
                : launch_pdl((const void*)k_dict_decode<1, false>, grid, block, 0, stream, args);
}

cudaError_t launch_dict_decode(const dictproj_group* g, const __half* X, int M, int mp, float* Zpart,
                               const DictPlan& plan, cudaStream_t stream) {
  return launch_dict_decode_batch(1, &g, &X, M, mp, &Zpart, &plan, stream);
}

bool decode_batch_gathers(int n, const dictproj_layer* const* l) {
  bool all = true;  // (bitmap and block layers have gather_ok false: one launch each)
  for (int i = 0; i < n; ++i) all = all && l[i]->gather_ok;
  return all;
}

// Time of a projection's CTAs in the gather kernel, in units of one 256-entry
// window of one warp: a warp takes whole columns, ceil(ceil(columns / CTAs) / 32)
// of them, and a column costs a fixed part worth two windows (its loads and
// addresses, the reduction and store; 1.06 us against 0.52 us per window,
// measured on B200) plus its windows, ceil(entries per column / 256).
static double gather_cta_time(size_t entries, int columns, int ctas, bool quantised) {
  const size_t epc = (entries + (size_t)std::max(1, columns) - 1) / (size_t)std::max(1, columns);
  const double cost = 2.0 + (double)((epc + 255) / 256);
  if (!quantised) return (double)columns / ctas / kGatherWarps * cost;
  const int cols = (columns + ctas - 1) / ctas;
  return (double)((cols + kGatherWarps - 1) / kGatherWarps) * cost;
}

void gather_batch_shares(int n, const size_t* entries, const int* columns, int n_sm, int* share) {
  // CTAs of a batched gather launch: one each, then one at a time to the
  // projection that would finish last (largest quantised time, then largest
  // smooth time), so that the launch ends as early as the cost allows; n_sm in all
  for (int i = 0; i < n; ++i) share[i] = 1;
  for (int given = n; given < n_sm; ++given) {
    int worst = 0;
    double wq = -1.0, ws = -1.0;
    for (int i = 0; i < n; ++i) {
      const double q = gather_cta_time(entries[i], columns[i], share[i], true);
      const double sm = gather_cta_time(entries[i], columns[i], share[i], false);
      if (q > wq || (q == wq && sm > ws)) worst = i, wq = q, ws = sm;
    }
    ++share[worst];
  }
}

static cudaError_t launch_gather_batch(int n, const dictproj_layer* const* l, const float* const* Zpart,
                                       const int* nslices, int M, int mp, __half* const* Y, cudaStream_t stream) {
  CoeffBatch b{};
  b.n = n;
  b.M = M;
  int blocks = 0, kmax = 0;
  size_t entries[kMaxBatch];
  int columns[kMaxBatch], share[kMaxBatch];
  for (int i = 0; i < n; ++i) entries[i] = l[i]->total, columns[i] = l[i]->d_out;
  gather_batch_shares(n, entries, columns, l[0]->n_sm, share);
  for (int i = 0; i < n; ++i) {
    CoeffProj& p = b.p[i];
    p.col_ptr = l[i]->col_ptr;
    p.codes = l[i]->codes;
    p.scales = l[i]->scales;
    p.idx = l[i]->idx;
    p.seg_start = l[i]->seg_start;
    p.nseg = l[i]->nseg;
    p.k = l[i]->k;
    p.d_out = l[i]->d_out;
    p.s = l[i]->s;
    p.Zpart = Zpart[i];
    p.nslices = nslices[i];
    p.Y = Y[i];
    const int ctas = share[i];
    p.cols_per_cta = (p.d_out + ctas - 1) / ctas;
    p.block_begin = blocks;
    blocks += (p.d_out + p.cols_per_cta - 1) / p.cols_per_cta;
    kmax = std::max(kmax, p.k);
  }
  void* args[] = {(void*)&b};
  const dim3 grid(blocks), block(kGatherWarps * 32);
  const size_t smem = (size_t)(kmax + 256) * mp * sizeof(__half);
  switch (mp) {
    case 1: return launch_pdl((const void*)k_coeff_gather<1>, grid, block, smem, stream, args);
    case 2: return launch_pdl((const void*)k_coeff_gather<2>, grid, block, smem, stream, args);
    case 4: return launch_pdl((const void*)k_coeff_gather<4>, grid, block, smem, stream, args);
    default: return launch_pdl((const void*)k_coeff_gather<8>, grid, block, smem, stream, args);
  }
}

cudaError_t launch_coeff_decode_batch(int n, const dictproj_layer* const* l, const float* const* Zpart,
                                      const int* nslices, int M, int mp, __half* const* Y, cudaStream_t stream) {
  if (decode_batch_gathers(n, l)) return launch_gather_batch(n, l, Zpart, nslices, M, mp, Y, stream);
  for (int i = 0; i < n; ++i) {
    cudaError_t e = launch_coeff_decode(l[i], Zpart[i], nslices[i], M, mp, Y[i], stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_coeff_decode(const dictproj_layer* l, const float* Zpart, int nslices, int M, int mp,
                                __half* Y, cudaStream_t stream) {
  if (l->ifmt != DICTPROJ_IFMT_U8) return launch_coeff_index(l, Zpart, nslices, M, mp, Y, stream);
  const uint8_t* codes = l->codes;
  const uint8_t* scales = l->scales;
  const uint8_t* idx = l->idx;
  const uint16_t* ss = l->seg_start;
  int nseg = l->nseg;
  float s = l->s;
  int k = l->k, d_out = l->d_out;
  if (l->gather_ok) return launch_gather_batch(1, &l, &Zpart, &nslices, M, mp, &Y, stream);
  const uint32_t* col_ptr = l->col_ptr;
  void* args[] = {(void*)&col_ptr, (void*)&codes, (void*)&scales, (void*)&idx, (void*)&ss,
                  (void*)&nseg, (void*)&s, (void*)&k, (void*)&d_out, (void*)&Zpart, (void*)&nslices,
                  (void*)&M, (void*)&Y};
  const dim3 grid((d_out + 7) / 8), block(256);
  const size_t smem = (size_t)(k + 256) * mp * sizeof(float);
  switch (mp) {
    case 1: return launch_pdl((const void*)k_coeff_decode_direct<1>, grid, block, smem, stream, args);
    case 2: return launch_pdl((const void*)k_coeff_decode_direct<2>, grid, block, smem, stream, args);
    case 4: return launch_pdl((const void*)k_coeff_decode_direct<4>, grid, block, smem, stream, args);
    default: return launch_pdl((const void*)k_coeff_decode_direct<8>, grid, block, smem, stream, args);
  }
}

bool gather_supported(const uint32_t* pcol_ptr, int d_out, int nseg) {
  if (nseg > 32) return false;
  for (int o = 0; o < d_out; ++o)
    if (pcol_ptr[o + 1] - pcol_ptr[o] > (uint32_t)(kRmax * 256)) return false;
  return true;
}

// Self-test of the bounded-wait error path: one warp waits on an mbarrier that
// expects two arrivals and receives one, so the wait can only end by its limit
// of `cycles` SM clocks. Nothing else is in flight when it gives up.
__global__ void k_wait_probe(long long cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    uint64_t state;
    asm volatile("mbarrier.arrive.shared::cta.b64 %0, [%1];" : "=l"(state) : "r"(smem_u32(&bar)) : "memory");
    (void)state;
    mbar_wait_bounded(&bar, 0, cycles);
  }
  __syncwarp();
}

cudaError_t launch_wait_probe(long long cycles, cudaStream_t stream) {
  k_wait_probe<<<1, 32, 0, stream>>>(cycles);
  return cudaGetLastError();
}

cudaError_t set_gather_times(unsigned long long* buf, int max_ctas) {
  cudaError_t e = cudaMemcpyToSymbol(g_gather_times, &buf, sizeof(buf));
  if (e != cudaSuccess) return e;
  const int n = buf ? max_ctas : 0;
  return cudaMemcpyToSymbol(g_gather_ctas, &n, sizeof(n));
}

cudaError_t take_decode_error(unsigned int* out) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_dictproj_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_dictproj_error, &zero, sizeof(unsigned int));
}

}  // namespace dictproj
