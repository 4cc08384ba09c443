// Decode path (M <= 8 tokens), fused: both stages of Eq. (1) of the DictLLM
// technical review, Z = X D_g and Y = Z C_l, in ONE kernel per call
// (k_decode_fused), with every packed weight byte staged through shared memory
// by bulk asynchronous copies.
//
// Why one kernel. At decode a projection moves 9-25 MB of packed weights, which
// HBM delivers in 1.3-3.7 us; two dependent kernels per call with a global Z
// round trip cost more than that in fixed latency. Here:
//   * one CTA per SM (grid = SM count); a producer warp streams the CTA's share
//     of the packed D_g and C_l into a ring of 16 KB shared-memory slots with
//     cp.async.bulk. Weights are never written after upload, so the producer
//     starts streaming at once, before the kernel waits for the previous work on
//     the stream (programmatic dependent launch): the ring of the next call
//     fills while this call computes. A CTA uses at most half of an SM (M <= 4),
//     so two consecutive calls are resident together.
//   * D_g is also kept in a tile-major copy made at upload: 16 atoms x 512
//     elements ("pieces") of codes (4 KB, 16-byte chunks of each row swizzled by
//     the row number, so that the MMA operand reads are conflict-free) and of
//     scales (512 B) are contiguous, and a CTA's share of a projection (a run of
//     consecutive pieces) is one contiguous range: one copy per slot.
//   * stage 1: twelve compute warps take 128-element quarters of the pieces,
//     decode E2M1 x E4M3 to fp16 (exact) and run swap-AB mma.sync m16n8k16 (atoms
//     = the 16 rows, tokens = the 8 columns) with fp32 accumulation. Pieces are
//     dealt to CTAs evenly, so a 16-atom tile is split over at most a few CTAs;
//     each writes its partial sums (times s_D) to the group's exchange buffer
//     Zx[slot][k][mp], every value in one 64-bit store together with this
//     launch's tag for the buffer (from a 64-bit ticket every CTA takes per group
//     at start).
//   * the exchange is the read: each CTA loads every slot of every tile for its
//     Z table and retries a value until it carries this launch's tag; slots are
//     summed in a fixed order, so Z is bit-exact and independent of timing.
//   * stage 2: each half of a compute warp takes one column of the CTA's column
//     chunks of C_l (columns split over CTAs by bytes, so by nnz); its 16 lanes
//     take 8-entry half-blocks, the segment of each entry comes from per-window
//     ballots over seg_start, fp32 sums, fp16 Y.
// Every wait is bounded (a second by default); a wait that gives up sets the
// device error word and the CTA unwinds (the producer first waits, bounded,
// for its copies in flight).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {

// ---------------------------------------------------------------------------------
// geometry
// ---------------------------------------------------------------------------------
constexpr int kFWarps = 12;                      // compute warps
constexpr int kFThreads = 32 * (kFWarps + 1);    // + one producer warp
constexpr int kPieceElems = 512;                 // d_in elements of one D piece (per atom)
constexpr int kPieceCodeBytes = 16 * 256;        // 16 atoms x 256 code bytes
constexpr int kPieceScaleBytes = 16 * 32;        // 16 atoms x 32 scale bytes
constexpr int kPiecesPerSlot = 3;
constexpr int kSlotScaleOff = kPiecesPerSlot * kPieceCodeBytes;  // 12 KB
constexpr int kMaxCChunks = 64;                  // coefficient chunks one CTA may own in one launch
constexpr int kMaxDChunks = 64;                  // dictionary slots one CTA may own in one launch
constexpr int kFusedMaxBatch = 4;

static_assert(kSlotScaleOff + kPiecesPerSlot * kPieceScaleBytes <= kFusedSlotBytes, "D pieces fit a slot");

// Tile-major copy of a packed dictionary (host side, at upload). Piece x =
// (tile a, piece pc of the atom row) holds rows r = 0..15 (atom 16a + r),
// elements [512 pc, 512 pc + 512): codes at x*4096 + r*256, the 16-byte chunk c of
// the row stored at position (c & 8) | ((c & 7) ^ (r & 7)); scales at x*512 + r*32.
// Elements at or beyond d_in are zero.
void fused_pack_dictionary(const uint8_t* codes, const uint8_t* scales, int d_in, int k, uint8_t* fcodes,
                           uint8_t* fscales) {
  const int ppr = (d_in + kPieceElems - 1) / kPieceElems;
  const size_t crow = (size_t)d_in / 2, srow = (size_t)d_in / 16;
  for (int a = 0; a < k / 16; ++a)
    for (int pc = 0; pc < ppr; ++pc) {
      const size_t x = (size_t)a * ppr + pc;
      for (int r = 0; r < 16; ++r) {
        const size_t atom = (size_t)16 * a + r;
        for (int c = 0; c < 16; ++c) {
          const int pos = (c & 8) | ((c & 7) ^ (r & 7));
          uint8_t* dst = fcodes + x * kPieceCodeBytes + r * 256 + pos * 16;
          for (int i = 0; i < 16; ++i) {
            const size_t byte = (size_t)pc * 256 + c * 16 + i;
            dst[i] = byte < crow ? codes[atom * crow + byte] : 0;
          }
        }
        for (int i = 0; i < 32; ++i) {
          const size_t byte = (size_t)pc * 32 + i;
          fscales[x * kPieceScaleBytes + r * 32 + i] = byte < srow ? scales[atom * srow + byte] : 0;
        }
      }
    }
}

// Byte layout of one coefficient chunk (columns [o_a, o_b), entries [E_a, E_b))
// in a ring slot: five 16-byte aligned runs copied from the packed arrays, each
// rounded outward to 16 bytes (the arrays carry 16 bytes of slack at the end).
struct CChunk {
  uint32_t idx_src, idx_bytes;    // idx[E_a, E_b)
  uint32_t code_src, code_bytes;  // values: codes[E_a*v/2, E_b*v/2) for v nibbles per value
  uint32_t sc_src, sc_bytes;      // scales[E_a/16, E_b/16) (NVFP4 only)
  uint32_t ss_src, ss_bytes;      // seg_start rows o_a .. o_b-1 (bytes)
  uint32_t cp_src, cp_bytes;      // col_ptr[o_a .. o_b] (bytes)
  uint32_t code_dst, sc_dst, ss_dst, cp_dst, total;
};

__host__ __device__ inline uint32_t up16(uint32_t x) { return (x + 15u) & ~15u; }

// Nibbles of one stored coefficient value: NVFP4 1 (plus a scale byte per 16),
// FP8 / INT8 2, FP16 4.
__host__ __device__ inline uint32_t cfmt_nibbles(int fmt) { return fmt == 0 ? 1u : fmt == 1 ? 4u : 2u; }

__host__ __device__ inline CChunk c_chunk_layout(uint32_t o_a, uint32_t o_b, uint32_t E_a, uint32_t E_b,
                                                 uint32_t nseg, int fmt) {
  const uint32_t vn = cfmt_nibbles(fmt);
  CChunk c;
  c.idx_src = E_a;
  c.idx_bytes = E_b - E_a;
  c.code_src = ((E_a * vn) >> 1) & ~15u;
  c.code_bytes = up16((E_b * vn) >> 1) - c.code_src;
  c.sc_src = fmt == 0 ? (E_a >> 4) & ~15u : 0u;
  c.sc_bytes = fmt == 0 ? up16(E_b >> 4) - c.sc_src : 0u;
  c.ss_src = (2u * o_a * nseg) & ~15u;
  c.ss_bytes = up16(2u * o_b * nseg) - c.ss_src;
  c.cp_src = (4u * o_a) & ~15u;
  c.cp_bytes = up16(4u * (o_b + 1u)) - c.cp_src;
  c.code_dst = c.idx_bytes;
  c.sc_dst = c.code_dst + c.code_bytes;
  c.ss_dst = c.sc_dst + c.sc_bytes;
  c.cp_dst = c.ss_dst + c.ss_bytes;
  c.total = c.cp_dst + c.cp_bytes;
  return c;
}

// Even split of P pieces over G positions: position c gets
// [c*q + min(c, r), (c+1)*q + min(c+1, r)) with P = q*G + r.
__host__ __device__ inline int split_begin(int c, int q, int r) { return c * q + (c < r ? c : r); }
__host__ __device__ inline int split_pos(int x, int q, int r) {
  return x < r * (q + 1) ? x / (q + 1) : r + (x - r * (q + 1)) / q;
}

// ---------------------------------------------------------------------------------
// launch parameters
// ---------------------------------------------------------------------------------
struct FusedProj {
  const uint8_t* fcodes;      // tile-major dictionary codes [P][4096]
  const uint8_t* fscales;     // tile-major dictionary scales [P][512]
  const __half* X;
  __half* Y;
  unsigned long long* zx;     // [zslots][k][MP]: (tag << 32) | fp32 bits of a tile piece's partial Z
  unsigned long long* ticket; // this group's launch ticket (one per CTA per launch)
  const uint32_t* col_ptr;
  const uint8_t* ccodes;
  const uint8_t* cscales;
  const uint8_t* cidx;
  const uint16_t* seg_start;
  const uint32_t* cplan_off;  // [G+1] first coefficient chunk of each position
  const uint4* cplan;         // chunks {o_a, o_b, E_a, E_b}
  float s_D, s_C;
  int d_in, k, d_out, nseg;
  int ppr, P, pq, pr, rot;    // pieces per atom row, pieces, P = pq*G + pr, position rotation
  int cfmt;                   // coefficient value format (DICTPROJ_CFMT_*)
  int xoff;                   // byte offset of its staged X rows in shared memory, -1: read X from global
  int xfirst;                 // 1: this projection stages X at xoff (later ones with the same X reuse it)
  int zt_off;                 // byte offset of its Z table in shared memory
  int zslots;                 // slots of the exchange buffer
};

struct FusedParams {
  FusedProj p[kFusedMaxBatch];
  long long wait_limit;        // SM clocks a bounded wait may take
  int n, M, G, R;              // projections, tokens, CTAs, ring slots
  int xrow;                    // bytes per staged X row
  int red_off;                 // shared-memory offset of the per-warp partial sums
  int n_tp;                    // tile pieces the red area holds per CTA
  int zt_resident;             // 1: every projection's Z table is resident; 0: one table reloaded per projection
  int bar_off;                 // offset of the barriers and chunk descriptors
};

}  // namespace dictproj

namespace dictproj {

// ---------------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void sts_u32x4(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// Bounded wait on an mbarrier phase that also gives up when another warp of the
// CTA has aborted (*abort != 0). Returns false when it gave up.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t phase, volatile int* abort,
                                                   long long limit) {
  if (mbar_try_wait(bar, phase)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, phase)) {
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      atomicOr(&g_dictproj_error, 1u);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// Diagnostic: wall-clock (ns) at the phase boundaries of the last fused launch,
// per CTA (slots 0-7 compute side, 8-11 producer side); read by
// dictproj_diag_phase_times. A few stores per CTA and launch.
constexpr int kPhaseCtas = 1024, kPhaseSlots = 16;
static __device__ unsigned long long g_phase[kPhaseCtas * kPhaseSlots];
__device__ __forceinline__ void phase_mark(int cta, int slot) {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  if (cta < kPhaseCtas) g_phase[cta * kPhaseSlots + slot] = t;
}

// ---------------------------------------------------------------------------------
// stage 1: one 16-atom x 128-element quarter of a D piece
// ---------------------------------------------------------------------------------
// Thread (g, tq) of the warp takes the 16-byte chunk c16 = 2*tq + h of box b of
// the atom rows g and g+8 (rows of 256 bytes; chunk c of row r stored at
// (c & 8) | ((c & 7) ^ (r & 7))), i.e. 32 elements per atom, and the same 32
// elements of X for token g. mma.sync m16n8k16 with the atoms as the 16 rows of A
// and the tokens as the 8 columns of B: within each thread the same element
// order is used for A and B, so the sum over k is unchanged.
__device__ __forceinline__ void piece_quarter(float acc[2][4], uint32_t box, uint32_t scl, int g, int c16,
                                              const uint32_t xw[4][4]) {
  const uint32_t ra = box + g * 256 + ((uint32_t)(c16 ^ g) << 4);
  const uint4 wa4 = lds_u32x4(ra), wb4 = lds_u32x4(ra + 2048);
  const uint32_t ha = e4m3x2_to_f16x2(lds_u16(scl + g * 32 + 2 * c16));
  const uint32_t hb = e4m3x2_to_f16x2(lds_u16(scl + (g + 8) * 32 + 2 * c16));
  const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
  const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
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
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a[4] = {fa[2 * h], fb[2 * h], fa[2 * h + 1], fb[2 * h + 1]};
      const uint32_t b[2] = {xw[q][2 * h], xw[q][2 * h + 1]};
      mma_16816(acc[h], a, b);
    }
  }
}

// ---------------------------------------------------------------------------------
// stage 2: coefficient values and one column from a shared-memory chunk
// ---------------------------------------------------------------------------------
// Eight stored values of half-block hb as four f16x2 (their fp16 forms are
// exact: E2M1, E4M3 and small integers are fp16 numbers), for each format.
template <int FMT>
__device__ __forceinline__ void half_block_values(uint32_t code_a, int hb, uint32_t f[4]) {
  if constexpr (FMT == 0) {  // NVFP4: 8 nibbles
    e2m1x8_to_f16x2x4(lds_u32(code_a + 4 * hb), f);
  } else if constexpr (FMT == 1) {  // FP16
    const uint4 v = lds_u32x4(code_a + 16 * hb);
    f[0] = v.x;
    f[1] = v.y;
    f[2] = v.z;
    f[3] = v.w;
  } else if constexpr (FMT == 2) {  // FP8 E4M3
    const uint2 v = lds_u32x2(code_a + 8 * hb);
    f[0] = e4m3x2_to_f16x2(v.x & 0xFFFF);
    f[1] = e4m3x2_to_f16x2(v.x >> 16);
    f[2] = e4m3x2_to_f16x2(v.y & 0xFFFF);
    f[3] = e4m3x2_to_f16x2(v.y >> 16);
  } else {  // INT8: |code| <= 127 is exact in fp16
    const uint2 v = lds_u32x2(code_a + 8 * hb);
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t word = w[i >> 1];
      const int sh = 16 * (i & 1);
      const __half2 h = __floats2half2_rn((float)(int8_t)((word >> sh) & 0xFF),
                                          (float)(int8_t)((word >> (sh + 8)) & 0xFF));
      f[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
}

// Sum over the 8 entries q0 .. q0+7 of a half-block: at most one segment
// boundary inside (t: first entry in segment sgi+1) unless `walk`, in which case
// the entries advance through seg_start one by one. Unscaled (block scale and
// s_C are applied by the caller).
template <int MP, int FMT>
__device__ __forceinline__ void half_block_sum(float out[MP], uint32_t idx_a, uint32_t code_a, uint32_t ss_a,
                                               int hb, int q0, int sgi, int t1, bool walk, int nseg, uint32_t zs_a) {
  constexpr uint32_t kRow = MP * 4;
  const uint2 iv = lds_u32x2(idx_a + 8 * hb);
  const uint32_t iw[2] = {iv.x, iv.y};
  uint32_t f[4];
  half_block_values<FMT>(code_a, hb, f);
  float a0[MP], a1[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) a0[m] = a1[m] = 0.f;
  if (!walk) {
    // Entries e >= t lie in segment sgi + 1: a bump byte of 1 for them, paired with
    // the index byte by one byte permute, gives two 9-bit atom offsets from z0.
    const int t = min(t1 - q0, 8);
    const unsigned long long bump = t >= 8 ? 0ull : (~0ull << (8 * t)) & 0x0101010101010101ull;
    const uint32_t bw[2] = {(uint32_t)bump, (uint32_t)(bump >> 32)};
    const uint32_t z0 = zs_a + ((uint32_t)sgi << 8) * kRow;
    unsigned long long acc2 = 0ull;  // (even, odd) entry sums for MP == 1
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[p]));
      const int j0 = (2 * p) & 3, w = p >> 1;
      const uint32_t pr = __byte_perm(iw[w], bw[w], (uint32_t)(j0 | ((j0 + 4) << 4) | ((j0 + 1) << 8) | ((j0 + 5) << 12)));
      const uint32_t ad0 = z0 + (pr & 0xFFFFu) * kRow, ad1 = z0 + (pr >> 16) * kRow;
      if constexpr (MP == 1) {
        unsigned long long zz, vv;
        asm("mov.b64 %0, {%1, %2};" : "=l"(zz) : "f"(lds_f32(ad0)), "f"(lds_f32(ad1)));
        asm("mov.b64 %0, {%1, %2};" : "=l"(vv) : "f"(v.x), "f"(v.y));
        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc2) : "l"(zz), "l"(vv));
      } else {
        fma_z<MP>(a0, ad0, v.x);
        fma_z<MP>(a1, ad1, v.y);
      }
    }
    if constexpr (MP == 1) {
      float lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc2));
      a0[0] = lo;
      a1[0] = hi;
    }
  } else {
    int sg = 0;
    for (int j = 1; j < nseg; ++j) sg += ((int)lds_u16(ss_a + 2 * j) <= q0);
    int nb = (sg + 1 < nseg) ? (int)lds_u16(ss_a + 2 * (sg + 1)) : INT_MAX;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[p]));
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int ent = 2 * p + hh;
        while (q0 + ent >= nb) {
          ++sg;
          nb = (sg + 1 < nseg) ? (int)lds_u16(ss_a + 2 * (sg + 1)) : INT_MAX;
        }
        const uint32_t bb = __byte_perm(iw[ent >> 2], 0u, 0x4440u | (uint32_t)(ent & 3));
        fma_z<MP>(hh ? a1 : a0, zs_a + (((uint32_t)sg << 8) + bb) * kRow, hh ? v.y : v.x);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) out[m] = a0[m] + a1[m];
}

// One column by G lanes (G = 32: a warp; G = 16: half a warp, `half` 0 / 1) in
// windows of 8*G entries: lane l of the group takes half-block G*i + l. The
// segment of each half-block's first entry, and the first entry of the next
// segment inside it, come from ballots over seg_start (lane l holds
// seg_start[l], so nseg <= G); two boundaries inside one half-block make the
// whole window walk. Returns the column sum (unscaled by s_C) in every lane.
template <int MP, int FMT, int G>
__device__ __forceinline__ void column_sum(float acc[MP], uint32_t idx_a, uint32_t code_a, uint32_t sc_a,
                                           uint32_t ss_a, int nhb, int nseg, uint32_t zs_a, int lane, int half) {
  const unsigned gmask = G == 32 ? 0xffffffffu : (0xffffu << (16 * half));
  const int gl = G == 32 ? lane : lane & 15;
  const unsigned gsh = G == 32 ? 0u : 16u * half;
  const unsigned lowbits = G == 32 ? 0xffffffffu : 0xffffu;
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.f;
  const bool is_bnd = gl >= 1 && gl < nseg;
  const int b = gl < nseg ? (int)lds_u16(ss_a + 2 * gl) : 0;
  for (int i = 0; 8 * G * i < 8 * nhb; ++i) {
    const int w = 8 * G * i;
    const int s_lo = __popc((__ballot_sync(gmask, is_bnd && b <= w) >> gsh) & lowbits);
    const bool in_win = is_bnd && b > w && b < w + 8 * G;
    const int rel = b - w;
    const uint32_t at_start = (in_win && (rel & 7) == 0) ? (1u << (rel >> 3)) : 0u;
    const uint32_t inside = (in_win && (rel & 7) != 0) ? (1u << (rel >> 3)) : 0u;
    const uint32_t A = __reduce_or_sync(gmask, at_start);
    const uint32_t B = __reduce_or_sync(gmask, inside);
    const int nwin = __popc((__ballot_sync(gmask, in_win) >> gsh) & lowbits);
    const bool collide = nwin != __popc(A) + __popc(B) || (A & B) != 0u;
    const uint32_t le = gl == 31 ? 0xffffffffu : ((2u << gl) - 1u);
    const int sgi = s_lo + __popc(A & le) + __popc(B & (le >> 1));  // segment of the lane's first entry
    const int q0 = w + 8 * gl;
    const int bn = __shfl_sync(gmask, b, min(sgi + 1, G - 1), G);
    const int t1 = ((B >> gl) & 1u) ? bn : INT_MAX;
    const int hb = G * i + gl;
    if (hb < nhb) {
      float s8[MP];
      half_block_sum<MP, FMT>(s8, idx_a, code_a, ss_a, hb, q0, sgi, t1, collide, nseg, zs_a);
      if constexpr (FMT == 0) {
        const float sc = e4m3_to_f32(lds_u8(sc_a + (hb >> 1)));
#pragma unroll
        for (int m = 0; m < MP; ++m) acc[m] = fmaf(s8[m], sc, acc[m]);
      } else {
#pragma unroll
        for (int m = 0; m < MP; ++m) acc[m] += s8[m];
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) {
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(gmask, acc[m], off, G);
  }
}

}  // namespace dictproj

namespace dictproj {

// Shared-memory control block (at FusedParams::bar_off, 16-byte aligned):
//   uint4   desc[kMaxCChunks]      coefficient chunks {o_a, o_b, E_a, E_b} of this CTA
//   uint32  dtab[kMaxDChunks]      dictionary slots: first piece | pieces << 28 | projection << 30
//   u64     full[R], empty[R], rdy mbarriers (ring slot filled / drained; control block ready)
//   int     misc[16]               abort, coefficient chunks, D pieces, tile pieces, D slots,
//                                  exchange tags of the projections (8..11)
//   int     loc[4][8]              per projection: x0, x1, first local piece, first tile piece,
//                                  first tile, tiles, position
//   uint8   desc_p[kMaxCChunks]    projection of each coefficient chunk
constexpr int kCtlMisc = 16, kCtlLoc = 8;
inline int fused_ctl_bytes(int R) {
  return 16 * kMaxCChunks + 4 * kMaxDChunks + 16 * R + 8 + 4 * kCtlMisc + 4 * kCtlLoc * kFusedMaxBatch + kMaxCChunks;
}

// Tagged read of one exchange value: retry until it carries `tag` (bounded).
__device__ __forceinline__ float ll_value(const unsigned long long* p, unsigned long long x, uint32_t tag,
                                          volatile int* abort, long long limit) {
  if ((uint32_t)(x >> 32) != tag) {
    const long long t0 = clock64();
    do {
      if (*abort) return 0.f;
      if (clock64() - t0 > limit) {
        atomicOr(&g_dictproj_error, 1u);
        *abort = 1;
        return 0.f;
      }
      __nanosleep(64);
      x = ld_relaxed_u64(p);
    } while ((uint32_t)(x >> 32) != tag);
  }
  return __uint_as_float((uint32_t)(x & 0xffffffffull));
}

// Z table of a projection in shared memory: Z[atom][m] = sum, in slot order, of the
// tile's partial sums in the exchange buffer (each read waits for this launch's
// tag), then a zero tail of 256 atom rows (padding entries read it).
template <int MP>
__device__ __forceinline__ void load_ztable(const FusedProj& pp, uint32_t sbase, int tid, uint32_t tag,
                                            volatile int* abort, long long limit) {
  constexpr int NT = kFWarps * 32, B = 4, S = 4;
  const uint32_t zt = sbase + pp.zt_off;
  const int ne = pp.k * MP;
  const size_t stride = (size_t)pp.k * MP;
  for (int base = tid; base < ne; base += B * NT) {
    unsigned long long v[B][S];
    int ns[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {  // issue every load of the batch before using any
      const int e = base + i * NT;
      ns[i] = 0;
      if (e < ne) {
        const int a = (e / MP) >> 4;
        ns[i] = split_pos(a * pp.ppr + pp.ppr - 1, pp.pq, pp.pr) - split_pos(a * pp.ppr, pp.pq, pp.pr) + 1;
      }
#pragma unroll
      for (int s = 0; s < S; ++s) v[i][s] = s < ns[i] ? ld_relaxed_u64(pp.zx + s * stride + e) : 0ull;
    }
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int e = base + i * NT;
      if (e >= ne) continue;
      float sum = 0.f;
#pragma unroll
      for (int s = 0; s < S; ++s)
        if (s < ns[i]) sum += ll_value(pp.zx + s * stride + e, v[i][s], tag, abort, limit);
      for (int s = S; s < ns[i]; ++s) {
        const unsigned long long* p = pp.zx + s * stride + e;
        sum += ll_value(p, ld_relaxed_u64(p), tag, abort, limit);
      }
      sts_f32(zt + 4 * e, sum);
    }
  }
  const int tail = (pp.k + 256) * MP;
  for (int v = ne + tid; v < tail; v += NT) sts_f32(zt + 4 * v, 0.f);
}

template <int MP>
__global__ void __launch_bounds__(kFThreads, 2) k_decode_fused(const __grid_constant__ FusedParams prm) {
  extern __shared__ uint8_t fsm_raw[];
  const uint32_t raw = smem_u32(fsm_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sg = fsm_raw + (sbase - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = prm.G, R = prm.R, n = prm.n, M = prm.M, cta = blockIdx.x;
  const long long limit = prm.wait_limit;
  uint4* desc = reinterpret_cast<uint4*>(sg + prm.bar_off);
  uint32_t* dtab = reinterpret_cast<uint32_t*>(desc + kMaxCChunks);
  uint64_t* full = reinterpret_cast<uint64_t*>(dtab + kMaxDChunks);
  uint64_t* empty = full + R;
  uint64_t* rdy = empty + R;
  int* misc = reinterpret_cast<int*>(rdy + 1);
  volatile int* s_abort = misc;
  int* loc = misc + kCtlMisc;
  uint8_t* desc_p = reinterpret_cast<uint8_t*>(loc + kCtlLoc * kFusedMaxBatch);

  if (threadIdx.x == kFWarps * 32) {
    for (int i = 0; i < R; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kFWarps);
    }
    mbar_init(rdy, 1);
    fence_mbar_init();
    int N1 = 0, ntp = 0, nD = 0;
    misc[0] = 0;
    for (int p = 0; p < n; ++p) {
      const FusedProj& pp = prm.p[p];
      int pos = cta - pp.rot;
      if (pos < 0) pos += G;
      const int x0 = split_begin(pos, pp.pq, pp.pr), x1 = split_begin(pos + 1, pp.pq, pp.pr);
      int* L = loc + kCtlLoc * p;
      L[0] = x0;
      L[1] = x1;
      L[2] = N1;
      L[3] = ntp;
      L[4] = x1 > x0 ? x0 / pp.ppr : 0;
      L[5] = x1 > x0 ? (x1 - 1) / pp.ppr - x0 / pp.ppr + 1 : 0;
      L[6] = pos;
      for (int x = x0; x < x1; x += kPiecesPerSlot) {  // slots of this projection's pieces
        if (nD < kMaxDChunks)
          dtab[nD] = (uint32_t)x | ((uint32_t)min(kPiecesPerSlot, x1 - x) << 28) | ((uint32_t)p << 30);
        ++nD;
      }
      N1 += x1 - x0;
      ntp += L[5];
    }
    misc[1] = 0;
    misc[2] = N1;
    misc[3] = ntp;
    misc[4] = nD;
    if (ntp > prm.n_tp || nD > kMaxDChunks) {  // the launcher checks both bounds: refuse rather than overrun
      atomicOr(&g_dictproj_error, 2u);
      misc[0] = 1;
      misc[4] = 0;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) phase_mark(cta, 0);
  const int nD = misc[4];

  if (warp == kFWarps) {
    // ------------------------------------------------------------- producer warp
    unsigned long long tk = 0;
    if (lane < n) tk = atomicAdd(prm.p[lane].ticket, 1ull);  // before any dependent grid may start
    auto issue = [&](int j) {
      const int s = j % R;
      const uint32_t dst = sbase + (uint32_t)s * kFusedSlotBytes;
      if (j < nD) {
        const uint32_t d = dtab[j];
        const int x = (int)(d & 0x0fffffffu), np = (int)((d >> 28) & 3u);
        const FusedProj& pp = prm.p[d >> 30];
        mbar_arrive_expect_tx(full + s, (uint32_t)np * (kPieceCodeBytes + kPieceScaleBytes));
        bulk_g2s_u32(dst, pp.fcodes + (size_t)x * kPieceCodeBytes, (uint32_t)np * kPieceCodeBytes, full + s);
        bulk_g2s_u32(dst + kSlotScaleOff, pp.fscales + (size_t)x * kPieceScaleBytes, (uint32_t)np * kPieceScaleBytes,
                     full + s);
      } else {
        const int t = j - nD;
        const uint4 d = desc[t];
        const FusedProj& pp = prm.p[desc_p[t]];
        const CChunk c = c_chunk_layout(d.x, d.y, d.z, d.w, (uint32_t)pp.nseg, pp.cfmt);
        mbar_arrive_expect_tx(full + s, c.total);
        if (c.idx_bytes) bulk_g2s_u32(dst, pp.cidx + c.idx_src, c.idx_bytes, full + s);
        if (c.code_bytes) bulk_g2s_u32(dst + c.code_dst, pp.ccodes + c.code_src, c.code_bytes, full + s);
        if (c.sc_bytes) bulk_g2s_u32(dst + c.sc_dst, pp.cscales + c.sc_src, c.sc_bytes, full + s);
        if (c.ss_bytes)
          bulk_g2s_u32(dst + c.ss_dst, reinterpret_cast<const uint8_t*>(pp.seg_start) + c.ss_src, c.ss_bytes, full + s);
        bulk_g2s_u32(dst + c.cp_dst, reinterpret_cast<const uint8_t*>(pp.col_ptr) + c.cp_src, c.cp_bytes, full + s);
      }
    };
    int issued = 0;
    if (lane == 0 && !*s_abort) {  // the first slots are free: start streaming D at once
      issued = min(R, nD);
      for (int j = 0; j < issued; ++j) issue(j);
      phase_mark(cta, 8);
    }
    // coefficient chunks of this CTA (position = CTA index) over all projections
    int beg = 0, cnt = 0;
    if (lane < n) {
      const uint32_t* off = prm.p[lane].cplan_off;
      beg = (int)off[cta];
      cnt = (int)off[cta + 1] - beg;
    }
    int pre = cnt;  // inclusive prefix over the lanes (projections)
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, pre, d);
      if (lane >= d) pre += v;
    }
    int ex[kFusedMaxBatch], bg[kFusedMaxBatch];
#pragma unroll
    for (int q = 0; q < kFusedMaxBatch; ++q) {
      ex[q] = __shfl_sync(0xffffffffu, pre - cnt, q);
      bg[q] = __shfl_sync(0xffffffffu, beg, q);
    }
    const int total_raw = __shfl_sync(0xffffffffu, pre, n - 1);
    const int total = total_raw > kMaxCChunks ? 0 : total_raw;
    for (int t = lane; t < total; t += 32) {
      int p = 0, b0 = bg[0], e0 = ex[0];
#pragma unroll
      for (int q = 1; q < kFusedMaxBatch; ++q)
        if (q < n && t >= ex[q]) {
          p = q;
          b0 = bg[q];
          e0 = ex[q];
        }
      desc[t] = prm.p[p].cplan[b0 + t - e0];
      desc_p[t] = (uint8_t)p;
    }
    if (lane < n) misc[8 + lane] = (int)((uint32_t)(tk / (unsigned long long)G) + 1u);  // exchange tags
    __syncwarp();
    if (lane == 0) {
      if (total_raw > kMaxCChunks) {  // the launcher checks this bound; refuse rather than drop chunks
        atomicOr(&g_dictproj_error, 2u);
        *s_abort = 1;
      }
      misc[1] = total;
      mbar_arrive_cta(rdy);
      trigger_dependents();
      phase_mark(cta, 9);
      // Slots are freed only by the compute warps, which first wait for the
      // previous grid on the stream; wait for it here too, so that the bounded
      // waits below measure this kernel's own progress, however long that grid runs.
      grid_dependency_wait();
      phase_mark(cta, 10);
      const int nall = nD + total;
      for (int j = issued; j < nall; ++j) {
        const int s = j % R;
        if (j >= R && !mbar_wait_or_abort(empty + s, (uint32_t)(((j / R) + 1) & 1), s_abort, limit)) break;
        if (*s_abort) break;
        issue(j);
        issued = j + 1;
      }
      phase_mark(cta, 11);
      if (*s_abort)  // let the copies in flight land before the CTA exits
        for (int j = max(0, issued - R); j < issued; ++j) mbar_wait_bounded(full + j % R, (uint32_t)((j / R) & 1), limit);
    }
  } else {
    // ------------------------------------------------------------- compute warps
    const int tid = threadIdx.x;
    const int g = lane >> 2, tq = lane & 3;
    grid_dependency_wait();  // X, the exchange buffer and Y belong to earlier work on the stream
    if (tid == 0) phase_mark(cta, 1);
    for (int i = tid; i < prm.n_tp * kFWarps * 16 * MP; i += kFWarps * 32) sts_f32(sbase + prm.red_off + 4 * i, 0.f);
    for (int p = 0; p < n; ++p) {  // stage X rows (element order permuted within 512-byte blocks)
      const FusedProj& pp = prm.p[p];
      if (pp.xoff < 0 || !pp.xfirst) continue;
      const int vpr = pp.ppr * 64;
      for (int v = tid; v < M * vpr; v += kFWarps * 32) {
        const int m = v / vpr, e = 8 * (v - m * vpr);
        const uint32_t dst = sbase + pp.xoff + m * prm.xrow + (e >> 8) * 512 + ((e >> 3) & 3) * 128 + ((e >> 5) & 7) * 16;
        const uint4 val = e < pp.d_in ? ld_cg_v4(pp.X + (size_t)m * pp.d_in + e) : make_uint4(0, 0, 0, 0);
        sts_u32x4(dst, val);
      }
    }
    named_bar_sync(1, kFWarps * 32);
    if (tid == 0) phase_mark(cta, 2);

    // ---- stage 1: partial Z of this CTA's D pieces
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int cur_tp = -1;
    auto flush = [&](int tp) {
      const uint32_t rb = sbase + prm.red_off + (uint32_t)((tp * kFWarps + warp) * 16 * MP) * 4;
      const int m0 = 2 * tq, m1 = 2 * tq + 1;
      if (m0 < MP) {
        sts_f32(rb + (g * MP + m0) * 4, acc[0][0] + acc[1][0]);
        sts_f32(rb + ((g + 8) * MP + m0) * 4, acc[0][2] + acc[1][2]);
      }
      if (m1 < MP) {
        sts_f32(rb + (g * MP + m1) * 4, acc[0][1] + acc[1][1]);
        sts_f32(rb + ((g + 8) * MP + m1) * 4, acc[0][3] + acc[1][3]);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;
    };
    for (int j = 0; j < nD; ++j) {
      const int s = j % R;
      bool ok = mbar_wait_or_abort(full + s, (uint32_t)((j / R) & 1), s_abort, limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      const uint32_t d = dtab[j];
      const int x_first = (int)(d & 0x0fffffffu), np = (int)((d >> 28) & 3u), p = (int)(d >> 30);
      const FusedProj& pp = prm.p[p];
      const uint32_t slot = sbase + (uint32_t)s * kFusedSlotBytes;
      for (int t = (warp + 4 * j) % kFWarps; t < 4 * np; t += kFWarps) {  // quarters round-robin, rotated per slot
        const int i = t >> 2, x = x_first + i;
        const int a = x / pp.ppr, pc = x - a * pp.ppr;
        const int tp = loc[kCtlLoc * p + 3] + a - loc[kCtlLoc * p + 4];
        if (tp != cur_tp) {
          if (cur_tp >= 0) flush(cur_tp);
          cur_tp = tp;
        }
        const int b = (t >> 1) & 1, h = t & 1, c16 = 2 * tq + h;
        uint32_t xw[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xw[q][0] = xw[q][1] = xw[q][2] = xw[q][3] = 0u;
        if (g < M) {
          if (pp.xoff >= 0) {
            const uint32_t xa = sbase + pp.xoff + g * prm.xrow + (2 * pc + b) * 512 + c16 * 16;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = lds_u32x4(xa + q * 128);
              xw[q][0] = v.x;
              xw[q][1] = v.y;
              xw[q][2] = v.z;
              xw[q][3] = v.w;
            }
          } else {
            const int e0 = pc * kPieceElems + b * 256 + 32 * c16;
            if (e0 < pp.d_in) {
              const __half* xp = pp.X + (size_t)g * pp.d_in + e0;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 v = ld_cg_v4(xp + 8 * q);
                xw[q][0] = v.x;
                xw[q][1] = v.y;
                xw[q][2] = v.z;
                xw[q][3] = v.w;
              }
            }
          }
        }
        piece_quarter(acc, slot + (uint32_t)i * kPieceCodeBytes + b * 128,
                      slot + kSlotScaleOff + (uint32_t)i * kPieceScaleBytes + b * 16, g, c16, xw);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cta(empty + s);
    }
    if (cur_tp >= 0) flush(cur_tp);
    named_bar_sync(1, kFWarps * 32);
    if (tid == 0) phase_mark(cta, 3);

    // ---- partial Z of each tile piece (sum over warps, times s_D), tagged, to the exchange buffer
    const bool ready = __all_sync(0xffffffffu, mbar_wait_or_abort(rdy, 0, s_abort, limit));
    const int ntp = misc[3];
    if (ready && !*s_abort) {
      for (int v = tid; v < ntp * 16 * MP; v += kFWarps * 32) {
        const int tp = v / (16 * MP), r = v - tp * 16 * MP;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) sum += lds_f32(sbase + prm.red_off + (uint32_t)((tp * kFWarps + w) * 16 * MP + r) * 4);
        int p = 0;
        for (int q = 0; q < n; ++q)
          if (tp >= loc[kCtlLoc * q + 3] && tp < loc[kCtlLoc * q + 3] + loc[kCtlLoc * q + 5]) p = q;
        const FusedProj& pp = prm.p[p];
        const int a = loc[kCtlLoc * p + 4] + tp - loc[kCtlLoc * p + 3];
        const int slot = loc[kCtlLoc * p + 6] - split_pos(a * pp.ppr, pp.pq, pp.pr);
        const unsigned long long word = ((unsigned long long)(uint32_t)misc[8 + p] << 32) |
                                        (unsigned long long)__float_as_uint(sum * pp.s_D);
        st_relaxed_u64(pp.zx + ((size_t)slot * pp.k + 16 * a) * MP + r, word);
      }
    }
    if (tid == 0) phase_mark(cta, 4);

    // ---- Z tables (the exchange: each value read waits for this launch's tag)
    const int N2 = misc[1];
    if (prm.zt_resident) {
      if (!*s_abort)
        for (int p = 0; p < n; ++p) load_ztable<MP>(prm.p[p], sbase, tid, (uint32_t)misc[8 + p], s_abort, limit);
      named_bar_sync(1, kFWarps * 32);
    }
    if (tid == 0) {
      phase_mark(cta, 5);
      phase_mark(cta, 6);
    }

    // ---- stage 2: Y = Z C over this CTA's column chunks, a column per half warp
    const int half = lane >> 4;
    int cur_p = -1;
    for (int i = 0; i < N2; ++i) {
      const int j = nD + i, s = j % R;
      const int p = desc_p[i];
      if (!prm.zt_resident && p != cur_p) {  // one Z table at a time: reload between projections
        named_bar_sync(1, kFWarps * 32);
        if (!*s_abort) load_ztable<MP>(prm.p[p], sbase, tid, (uint32_t)misc[8 + p], s_abort, limit);
        named_bar_sync(1, kFWarps * 32);
      }
      cur_p = p;
      bool ok = mbar_wait_or_abort(full + s, (uint32_t)((j / R) & 1), s_abort, limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      const FusedProj& pp = prm.p[p];
      const uint4 d = desc[i];
      const int fmt = pp.cfmt;
      const CChunk c = c_chunk_layout(d.x, d.y, d.z, d.w, (uint32_t)pp.nseg, fmt);
      const uint32_t vn = cfmt_nibbles(fmt);
      const uint32_t slot = sbase + (uint32_t)s * kFusedSlotBytes;
      const int ncols = (int)(d.y - d.x);
      const uint32_t zs = sbase + pp.zt_off;
      const bool halves = pp.nseg <= 16;  // a column per half warp needs the segment starts in 16 lanes
      const int per = halves ? 2 : 1;
      for (int t0 = ((warp + i) % kFWarps) * per; t0 < ncols; t0 += kFWarps * per) {
        const int t = t0 + (halves ? half : 0);
        if (t >= ncols) continue;  // (halves only: this half idles; the other half's ballots use its own mask)
        const uint32_t o = d.x + (uint32_t)t;
        const uint32_t cpa = slot + c.cp_dst + 4u * o - c.cp_src;
        const uint32_t e0 = lds_u32(cpa), e1 = lds_u32(cpa + 4);
        const uint32_t ia = slot + (e0 - d.z), ca = slot + c.code_dst + ((e0 * vn) >> 1) - c.code_src;
        const uint32_t sa = slot + c.sc_dst + (e0 >> 4) - c.sc_src;
        const uint32_t ssa = slot + c.ss_dst + 2u * o * (uint32_t)pp.nseg - c.ss_src;
        const int nhb = (int)((e1 - e0) >> 3);
        float y[MP];
        if (halves) {
          switch (fmt) {  // uniform over the chunk
            case 0: column_sum<MP, 0, 16>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, half); break;
            case 1: column_sum<MP, 1, 16>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, half); break;
            case 2: column_sum<MP, 2, 16>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, half); break;
            default: column_sum<MP, 3, 16>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, half); break;
          }
        } else {
          switch (fmt) {
            case 0: column_sum<MP, 0, 32>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, 0); break;
            case 1: column_sum<MP, 1, 32>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, 0); break;
            case 2: column_sum<MP, 2, 32>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, 0); break;
            default: column_sum<MP, 3, 32>(y, ia, ca, sa, ssa, nhb, pp.nseg, zs, lane, 0); break;
          }
        }
        if ((lane & (halves ? 15 : 31)) == 0) {
#pragma unroll
          for (int m = 0; m < MP; ++m)
            if (m < M) pp.Y[(size_t)m * pp.d_out + o] = __float2half_rn(y[m] * pp.s_C);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cta(empty + s);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) phase_mark(cta, 7);
}

}  // namespace dictproj

// =================================================================================
// host side
// =================================================================================
namespace dictproj {

static int fused_pieces_per_row(int d_in) { return (d_in + kPieceElems - 1) / kPieceElems; }

// Largest number of tiles one position's piece range spans, and the largest
// number of positions one tile is split over (the exchange buffer's slots).
static void fused_split_bounds(int tiles, int ppr, int G, int* tp_bound, int* slots) {
  const int P = tiles * ppr, q = P / G, r = P % G;
  int tb = 0, sl = 1;
  for (int c = 0; c < G; ++c) {
    const int x0 = split_begin(c, q, r), x1 = split_begin(c + 1, q, r);
    if (x1 > x0) tb = std::max(tb, (x1 - 1) / ppr - x0 / ppr + 1);
  }
  for (int a = 0; a < tiles; ++a)
    sl = std::max(sl, split_pos(a * ppr + ppr - 1, q, r) - split_pos(a * ppr, q, r) + 1);
  *tp_bound = tb;
  *slots = sl;
}

cudaError_t fused_group_setup(dictproj_group* g, const uint8_t* codes, const uint8_t* scales, bool* ok) {
  *ok = false;
  g->fused_ok = false;
  if (g->k > 8192) return cudaSuccess;  // the gather keeps the segment starts in one warp
  const int tiles = g->k / 16;
  g->ppr = fused_pieces_per_row(g->d_in);
  fused_split_bounds(tiles, g->ppr, g->n_sm, &g->tp_bound, &g->zslots);
  const size_t P = (size_t)tiles * g->ppr;
  std::vector<uint8_t> fc, fs;
  try {
    fc.resize(P * kPieceCodeBytes);
    fs.resize(P * kPieceScaleBytes);
  } catch (...) {
    return cudaErrorMemoryAllocation;
  }
  fused_pack_dictionary(codes, scales, g->d_in, g->k, fc.data(), fs.data());
  cudaError_t e;
  if ((e = cudaMalloc((void**)&g->fcodes, fc.size())) != cudaSuccess) return e;
  if ((e = cudaMalloc((void**)&g->fscales, fs.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpy(g->fcodes, fc.data(), fc.size(), cudaMemcpyHostToDevice)) != cudaSuccess) return e;
  if ((e = cudaMemcpy(g->fscales, fs.data(), fs.size(), cudaMemcpyHostToDevice)) != cudaSuccess) return e;
  const size_t zx_bytes = (size_t)g->zslots * g->k * kDecodeMaxTokens * sizeof(unsigned long long);
  if ((e = cudaMalloc((void**)&g->zx, zx_bytes)) != cudaSuccess) return e;
  if ((e = cudaMemset(g->zx, 0, zx_bytes)) != cudaSuccess) return e;  // tag 0: never a launch's tag
  if ((e = cudaMalloc((void**)&g->fsync, 16)) != cudaSuccess) return e;
  if ((e = cudaMemset(g->fsync, 0, 16)) != cudaSuccess) return e;
  g->fused_ok = true;
  *ok = true;
  return cudaSuccess;
}

bool fused_layer_plan(const uint32_t* pcol_ptr, int d_out, int nseg, int fmt, int G, std::vector<uint32_t>& off,
                      std::vector<uint4>& chunks, int* max_per_pos) {
  off.assign(G + 1, 0);
  chunks.clear();
  *max_per_pos = 0;
  if (nseg > 32) return false;
  auto fits = [&](int oa, int ob) {
    return c_chunk_layout(oa, ob, pcol_ptr[oa], pcol_ptr[ob], nseg, fmt).total <= (uint32_t)kFusedSlotBytes;
  };
  // bytes streamed per column (balancing weight): index + values (+ scales) + seg_start + col_ptr
  const double per_entry = 1.0 + cfmt_nibbles(fmt) * 0.5 + (fmt == 0 ? 1.0 / 16 : 0.0);
  std::vector<double> cum(d_out + 1, 0.0);
  for (int o = 0; o < d_out; ++o) {
    const double ne = (double)(pcol_ptr[o + 1] - pcol_ptr[o]);
    cum[o + 1] = cum[o] + ne * per_entry + 2.0 * nseg + 4.0;
    if (!fits(o, o + 1)) return false;  // a column larger than a ring slot
  }
  auto lower = [&](int lo, int hi, double target) {  // first o in [lo, hi] with cum[o] >= target
    return (int)(std::lower_bound(cum.begin() + lo, cum.begin() + hi + 1, target) - cum.begin());
  };
  int o_lo = 0;
  for (int c = 0; c < G; ++c) {
    const int o_hi = c == G - 1 ? d_out : std::max(o_lo, lower(o_lo, d_out, cum[d_out] * (c + 1) / G));
    off[c] = (uint32_t)chunks.size();
    if (o_hi > o_lo) {
      int nch = 0;  // greedy count of slot-sized chunks
      for (int a = o_lo; a < o_hi; ++nch) {
        int b = a + 1;
        while (b < o_hi && fits(a, b + 1)) ++b;
        a = b;
      }
      // the same number of chunks, split evenly by bytes; greedy if one does not fit
      std::vector<int> cut(nch + 1);
      cut[0] = o_lo;
      cut[nch] = o_hi;
      bool even = true;
      for (int i = 1; i < nch; ++i) {
        const double t = cum[o_lo] + (cum[o_hi] - cum[o_lo]) * i / nch;
        cut[i] = std::min(o_hi - 1, std::max(cut[i - 1] + 1, lower(o_lo, o_hi, t)));
      }
      for (int i = 0; i < nch; ++i) even = even && cut[i + 1] > cut[i] && fits(cut[i], cut[i + 1]);
      if (!even) {
        cut.assign(1, o_lo);
        for (int a = o_lo; a < o_hi;) {
          int b = a + 1;
          while (b < o_hi && fits(a, b + 1)) ++b;
          cut.push_back(b);
          a = b;
        }
        nch = (int)cut.size() - 1;
      }
      for (int i = 0; i < nch; ++i)
        chunks.push_back(make_uint4((uint32_t)cut[i], (uint32_t)cut[i + 1], pcol_ptr[cut[i]], pcol_ptr[cut[i + 1]]));
      *max_per_pos = std::max(*max_per_pos, nch);
    }
    o_lo = o_hi;
  }
  off[G] = (uint32_t)chunks.size();
  return true;
}

cudaError_t fused_phase_times(unsigned long long* out, int max_ctas, int* n_ctas) {
  const int n = std::min(max_ctas, kPhaseCtas);
  *n_ctas = n;
  return cudaMemcpyFromSymbol(out, g_phase, (size_t)n * kPhaseSlots * sizeof(unsigned long long));
}

cudaError_t prepare_fused_kernels(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_decode_fused<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)) ||
      (e = cudaFuncSetAttribute(k_decode_fused<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)) ||
      (e = cudaFuncSetAttribute(k_decode_fused<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)) ||
      (e = cudaFuncSetAttribute(k_decode_fused<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin)))
    return e;
  return cudaSuccess;
}

// Shared memory per CTA for two CTAs to share an SM (228 KB, 1 KB reserved each).
constexpr int kCoResidentSmem = 113 * 1024;
constexpr int kStageXMax = 48 * 1024;

bool fused_plan_launch(int n, const dictproj_group* const* g, const dictproj_layer* const* l,
                       const __half* const* X, int M, int smem_optin, FusedLaunchPlan* out) {
  FusedLaunchPlan& pl = *out;
  pl = FusedLaunchPlan{};
  if (n < 1 || n > kFusedMaxBatch || M < 1 || M > kDecodeMaxTokens) return false;
  const int mp = decode_mp(M);
  int chunks = 0, tp = 0, max_ppr = 0, dslots = 0;
  for (int i = 0; i < n; ++i) {
    if (!g[i]->fused_ok || !l[i]->fused_ok || g[i]->n_sm != g[0]->n_sm || l[i]->n_sm != g[0]->n_sm) return false;
    chunks += l[i]->cplan_max;
    tp += g[i]->tp_bound;
    max_ppr = std::max(max_ppr, g[i]->ppr);
    const int P = (g[i]->k / 16) * g[i]->ppr;
    dslots += (P / g[i]->n_sm + 1 + kPiecesPerSlot - 1) / kPiecesPerSlot;
  }
  if (chunks > kMaxCChunks || dslots > kMaxDChunks) return false;
  pl.mp = mp;
  pl.n_tp = std::max(tp, 1);
  pl.xrow = max_ppr * 1024 + 16;
  // distinct activations are staged once
  int nx = 0, xtot = 0;
  for (int i = 0; i < n; ++i) {
    pl.xfirst[i] = 1;
    pl.xslot[i] = nx;
    for (int j = 0; j < i; ++j)
      if (X[j] == X[i] && g[j]->d_in == g[i]->d_in) {
        pl.xfirst[i] = 0;
        pl.xslot[i] = pl.xslot[j];
      }
    if (pl.xfirst[i]) ++nx;
  }
  xtot = M * pl.xrow * nx;
  pl.stage_x = xtot <= kStageXMax;
  const int red = pl.n_tp * kFWarps * 16 * mp * 4;
  const int stage1 = (pl.stage_x ? xtot : 0) + red;
  int zall = 0, zone = 0;
  for (int i = 0; i < n; ++i) {
    const int zb = (g[i]->k + 256) * mp * 4;
    zall += zb;
    zone = std::max(zone, zb);
  }
  auto total = [&](int R, int U) { return 1024 + R * kFusedSlotBytes + U + fused_ctl_bytes(R); };
  for (int pass = 0; pass < 2 && !pl.R; ++pass) {  // first: two CTAs per SM; then: one
    const int cap = pass == 0 ? kCoResidentSmem : smem_optin;
    const int rmin = pass == 0 ? 3 : 2;
    for (int resident = 1; resident >= 0 && !pl.R; --resident) {
      const int U = (std::max(stage1, resident ? zall : zone) + 15) & ~15;
      for (int R = 8; R >= rmin; --R)
        if (total(R, U) <= cap) {
          pl.R = R;
          pl.U = U;
          pl.zt_resident = resident;
          pl.smem = total(R, U);
          break;
        }
    }
  }
  if (!pl.R) return false;
  pl.red_off = pl.R * kFusedSlotBytes + (pl.stage_x ? xtot : 0);
  pl.bar_off = pl.R * kFusedSlotBytes + pl.U;
  int zo = pl.R * kFusedSlotBytes;
  for (int i = 0; i < n; ++i) {
    pl.xoff[i] = pl.stage_x ? pl.R * kFusedSlotBytes + pl.xslot[i] * M * pl.xrow : -1;
    pl.zt_off[i] = zo;
    if (pl.zt_resident) zo += (g[i]->k + 256) * mp * 4;
  }
  return true;
}

cudaError_t launch_fused(int n, const dictproj_group* const* g, const dictproj_layer* const* l,
                         const __half* const* X, __half* const* Y, int M, const FusedLaunchPlan& pl,
                         long long wait_limit, cudaStream_t stream) {
  FusedParams prm;
  memset(&prm, 0, sizeof(prm));
  const int G = g[0]->n_sm;
  int rot = 0;
  for (int i = 0; i < n; ++i) {
    FusedProj& p = prm.p[i];
    p.fcodes = g[i]->fcodes;
    p.fscales = g[i]->fscales;
    p.X = X[i];
    p.Y = Y[i];
    p.zx = g[i]->zx;
    p.ticket = g[i]->fsync;
    p.col_ptr = l[i]->col_ptr;
    p.ccodes = l[i]->codes;
    p.cscales = l[i]->scales;
    p.cidx = l[i]->idx;
    p.seg_start = l[i]->seg_start;
    p.cplan_off = l[i]->cplan_off;
    p.cplan = l[i]->cplan;
    p.cfmt = l[i]->cfmt;
    p.s_D = g[i]->s;
    p.s_C = l[i]->s;
    p.d_in = g[i]->d_in;
    p.k = g[i]->k;
    p.d_out = l[i]->d_out;
    p.nseg = l[i]->nseg;
    p.ppr = g[i]->ppr;
    p.P = (g[i]->k / 16) * p.ppr;
    p.pq = p.P / G;
    p.pr = p.P % G;
    p.rot = rot;
    rot = (rot + p.pr) % G;  // the next projection's larger shares go to the following CTAs
    p.xoff = pl.xoff[i];
    p.xfirst = pl.xfirst[i];
    p.zt_off = pl.zt_off[i];
    p.zslots = g[i]->zslots;
  }
  prm.wait_limit = wait_limit;
  prm.n = n;
  prm.M = M;
  prm.G = G;
  prm.R = pl.R;
  prm.xrow = pl.xrow;
  prm.red_off = pl.red_off;
  prm.n_tp = pl.n_tp;
  prm.zt_resident = pl.zt_resident;
  prm.bar_off = pl.bar_off;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (pl.mp) {
    case 1: return cudaLaunchKernelEx(&cfg, k_decode_fused<1>, prm);
    case 2: return cudaLaunchKernelEx(&cfg, k_decode_fused<2>, prm);
    case 4: return cudaLaunchKernelEx(&cfg, k_decode_fused<4>, prm);
    default: return cudaLaunchKernelEx(&cfg, k_decode_fused<8>, prm);
  }
}

}  // namespace dictproj
