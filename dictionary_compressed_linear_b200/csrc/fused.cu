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
#ifndef DICTPROJ_FUSED_COMPUTE_WARPS
#define DICTPROJ_FUSED_COMPUTE_WARPS 12
#endif
constexpr int kFWarps = DICTPROJ_FUSED_COMPUTE_WARPS;  // compute warps
constexpr int kFThreads = 32 * (kFWarps + 1);    // + one producer warp
constexpr int kPieceElems = 512;                 // d_in elements of one D piece (per atom)
constexpr int kPieceCodeBytes = 16 * 256;        // 16 atoms x 256 code bytes
constexpr int kPieceScaleBytes = 16 * 32;        // 16 atoms x 32 scale bytes
constexpr int kPiecesPerSlot = 3;
constexpr int kSlotScaleOff = kPiecesPerSlot * kPieceCodeBytes;  // 12 KB
constexpr int kMaxCChunks = 64;                  // coefficient chunks one CTA may own in one launch
constexpr int kMaxDChunks = 64;                  // dictionary slots one CTA may own in one launch
constexpr int kFusedMaxBatch = 4;
constexpr int kMaxStage2Batch = 4;                         // coefficient chunks per stage-2 batch

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
  int part_off;                // offset of the stage-2 partial sums (two buffers of 2 x threads x MP floats)
  int W;                       // coefficient chunks per stage-2 batch
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
// per CTA (slots 0-5 and 7 compute side, 8-11 producer side, 13 end of warp 0's
// stage 2), and as plain values: 6 and 12 ns warp 0 waited for dictionary slots
// and coefficient chunks, 14 coefficient chunks, 15 dictionary slots; read by
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
__device__ __forceinline__ void piece_quarter(float acc[4][4], uint32_t box, uint32_t scl, int g, int c16,
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
      mma_16816(acc[2 * (q & 1) + h], a, b);  // four accumulators: two MMAs in each chain
    }
  }
}

// ---------------------------------------------------------------------------------
// stage 2: coefficient values and one column from a shared-memory chunk
// ---------------------------------------------------------------------------------
// The stored values of half-block hb (8 entries) as raw words, and as four f16x2
// (their fp16 forms are exact: E2M1, E4M3 and small integers are fp16 numbers),
// for each format.
template <int FMT>
__device__ __forceinline__ uint4 hb_load(uint32_t code_a, int hb) {
  if constexpr (FMT == 0) {  // NVFP4: 8 nibbles
    return make_uint4(lds_u32(code_a + 4u * (uint32_t)hb), 0u, 0u, 0u);
  } else if constexpr (FMT == 1) {  // FP16
    return lds_u32x4(code_a + 16u * (uint32_t)hb);
  } else {  // FP8 / INT8
    const uint2 v = lds_u32x2(code_a + 8u * (uint32_t)hb);
    return make_uint4(v.x, v.y, 0u, 0u);
  }
}
template <int FMT>
__device__ __forceinline__ void hb_decode(uint4 r, uint32_t f[4]) {
  if constexpr (FMT == 0) {
    e2m1x8_to_f16x2x4(r.x, f);
  } else if constexpr (FMT == 1) {
    f[0] = r.x;
    f[1] = r.y;
    f[2] = r.z;
    f[3] = r.w;
  } else if constexpr (FMT == 2) {  // E4M3
    f[0] = e4m3x2_to_f16x2(r.x & 0xFFFF);
    f[1] = e4m3x2_to_f16x2(r.x >> 16);
    f[2] = e4m3x2_to_f16x2(r.y & 0xFFFF);
    f[3] = e4m3x2_to_f16x2(r.y >> 16);
  } else {  // INT8: |code| <= 127 is exact in fp16
    const uint32_t w[2] = {r.x, r.y};
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


// Segment state of a thread inside one column of C_l: sg is the segment of the
// current entry q (the number of segment starts s >= 1 with seg_start[s] <= q),
// nb and nb2 the next two segment starts (kSegNone past the last one).
constexpr int kSegNone = 1 << 30;
struct SegState {
  int sg, nb, nb2;
};
__device__ __forceinline__ int seg_at(uint32_t ssa, int s, int nseg) {
  return s < nseg ? (int)lds_u16(ssa + 2u * (uint32_t)s) : kSegNone;
}
__device__ __forceinline__ SegState seg_find(uint32_t ssa, int q, int nseg) {
  SegState st;
  st.sg = 0;
  for (int s = 1; s < nseg; ++s) st.sg += ((int)lds_u16(ssa + 2u * (uint32_t)s) <= q);
  st.nb = seg_at(ssa, st.sg + 1, nseg);
  st.nb2 = seg_at(ssa, st.sg + 2, nseg);
  return st;
}
// Move the state forward to the segment of entry q (segment starts only grow).
__device__ __forceinline__ void seg_advance(SegState& st, uint32_t ssa, int q, int nseg) {
  while (st.nb <= q) {
    ++st.sg;
    st.nb = st.nb2;
    st.nb2 = seg_at(ssa, st.sg + 2, nseg);
  }
}

// Sum over the 8 entries of a half-block (index bytes iv, values f) whose entries
// lie in at most two segments: entries e >= t belong to the segment `delta` after
// the one whose Z rows start at z0 (t >= 8: none). A bump byte of delta for those
// entries, paired with the index byte by one byte permute, gives two atom offsets
// from z0. Unscaled (block scale and s_C are applied by the caller).
// Sum over the 8 entries of a half-block (index bytes iv, values f) whose entries
// lie in at most two segments: entries e >= t belong to the segment after the one
// whose Z rows start at z0 (t >= 8: none). A bump byte of 1 for those entries,
// paired with the index byte by one byte permute, gives two atom offsets from z0.
// Unscaled (block scale and s_C are applied by the caller).
template <int MP>
__device__ __forceinline__ void hb_sum(float out[MP], uint2 iv, const uint32_t f[4], uint32_t z0, int t) {
  constexpr uint32_t kRow = MP * 4;
  const uint32_t iw[2] = {iv.x, iv.y};
  const uint32_t tt = (uint32_t)min(t, 8);  // entries tt..7 get a bump byte of 1
  const uint32_t bw[2] = {shl_clamped(0x01010101u, 8u * tt), shl_clamped(0x01010101u, 8u * (tt > 4u ? tt - 4u : 0u))};
  float a0[MP], a1[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) a0[m] = a1[m] = 0.f;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[p]));
    const int j0 = (2 * p) & 3, w = p >> 1;
    const uint32_t pr = __byte_perm(iw[w], bw[w], (uint32_t)(j0 | ((j0 + 4) << 4) | ((j0 + 1) << 8) | ((j0 + 5) << 12)));
    fma_z<MP>(a0, z0 + (pr & 0xFFFFu) * kRow, v.x);
    fma_z<MP>(a1, z0 + (pr >> 16) * kRow, v.y);
  }
#pragma unroll
  for (int m = 0; m < MP; ++m) out[m] = a0[m] + a1[m];
}

// The same sum when two or more segment starts lie inside the half-block: the
// segment advances entry by entry (q: column position of the first entry). Rare,
// so written as a plain loop to keep the hot loop's code small.
template <int MP>
__device__ __forceinline__ void hb_walk(float out[MP], uint2 iv, const uint32_t f[4], uint32_t zs, SegState& st,
                                        uint32_t ssa, int q, int nseg) {
  constexpr uint32_t kRow = MP * 4;
#pragma unroll
  for (int m = 0; m < MP; ++m) out[m] = 0.f;
#pragma unroll 1
  for (int ent = 0; ent < 8; ++ent) {
    seg_advance(st, ssa, q + ent, nseg);
    const uint32_t w = ent < 4 ? iv.x : iv.y;
    const uint32_t bb = (w >> (8 * (ent & 3))) & 0xFFu;
    const uint32_t fw = f[0];
    const uint32_t fp = ent < 2 ? fw : ent < 4 ? f[1] : ent < 6 ? f[2] : f[3];
    const float v = __half2float(__ushort_as_half((unsigned short)((ent & 1) ? fp >> 16 : fp & 0xFFFFu)));
    fma_z<MP>(out, zs + (((uint32_t)st.sg << 8) + bb) * kRow, v);
  }
}

// Stage 2 over a batch of resident coefficient chunks: the batch's half-blocks
// (chunk after chunk) are split evenly over the NL compute threads, thread L
// taking a contiguous run; stage2_run does the part of the run that lies in one
// chunk (columns [d.x, d.y), stored entries [d.z, d.w), in shared memory at
// `slot`; local half-blocks [h, h1)). Columns never cross chunks. A column that
// lies inside one run is finished by its thread (Y written); otherwise the thread
// leaves its share in the partial area `part`: HEAD (slot 0) for a column that
// began before its run, TAIL (slot 1) for one that began inside it and goes on
// after it, and then reports the column and its end (tail_o, tail_he): after the
// batch it adds the HEAD shares of the following threads to its TAIL, in order
// (the result does not depend on timing). Empty columns are written separately.
template <int MP, int FMT>
__device__ __forceinline__ void stage2_run(const FusedProj& pp, uint4 d, const CChunk& c, uint32_t slot,
                                           uint32_t zs, int h, int h1, int L, uint32_t part, int M, float yscale,
                                           int* tail_o, int* tail_he) {
  constexpr uint32_t kRow = MP * 4;
  if (h >= h1) return;
  const int nseg = pp.nseg;
  const uint32_t cpa = slot + c.cp_dst - c.cp_src;  // col_ptr[o] at cpa + 4 o
  const uint32_t ssb = slot + c.ss_dst - c.ss_src;  // seg_start row of column o at ssb + 2 o nseg
  const uint32_t ca = slot + c.code_dst + ((d.z * cfmt_nibbles(FMT)) >> 1) - c.code_src;
  const uint32_t sa = slot + c.sc_dst + (d.z >> 4) - c.sc_src;
  const uint32_t E0 = d.z + 8u * (uint32_t)h;
  int lo = (int)d.x, hi = (int)d.y - 1;  // the column holding entry E0: last o with col_ptr[o] <= E0
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (lds_u32(cpa + 4u * (uint32_t)mid) <= E0) lo = mid;
    else hi = mid - 1;
  }
  int o = lo;
  uint32_t cb = lds_u32(cpa + 4u * (uint32_t)o), ce = lds_u32(cpa + 4u * (uint32_t)o + 4u);
  bool started = cb == E0;
  int he = (int)((ce - d.z) >> 3);  // first half-block after column o
  int q = (int)(E0 - cb);           // column position of the half-block's first entry
  uint32_t ssa = ssb + 2u * (uint32_t)o * (uint32_t)nseg;
  SegState st = seg_find(ssa, q, nseg);
  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.f;
  // A column that ends inside the run is finished by its thread: written to Y if it
  // also began there, else left as HEAD.
  auto finish = [&]() {
    if (started) {
#pragma unroll
      for (int m = 0; m < MP; ++m)
        if (m < M) pp.Y[(size_t)m * pp.d_out + o] = __float2half_rn(acc[m] * yscale);
    } else {
      const uint32_t pa = part + (uint32_t)(2 * L * MP) * 4u;
#pragma unroll
      for (int m = 0; m < MP; ++m) sts_f32(pa + 4u * m, acc[m]);
    }
  };
  // One loop over the run's half-blocks for every thread of the warp; a column
  // change is a short branch inside it.
  for (; h < h1; ++h, q += 8) {
    if (h == he) {
      finish();
      do {  // the next column with entries (empty columns are written by stage2_combine)
        ++o;
        cb = ce;
        ce = lds_u32(cpa + 4u * (uint32_t)o + 4u);
      } while (ce == cb);
      he = (int)((ce - d.z) >> 3);
      started = true;
      q = 0;
      ssa = ssb + 2u * (uint32_t)o * (uint32_t)nseg;
      st = seg_find(ssa, 0, nseg);
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] = 0.f;
    }
    const uint2 iv = lds_u32x2(slot + 8u * (uint32_t)h);
    uint32_t f[4];
    hb_decode<FMT>(hb_load<FMT>(ca, h), f);
    float s8[MP];
    if (st.nb2 < q + 8) {  // three or more segments (rare)
      hb_walk<MP>(s8, iv, f, zs, st, ssa, q, nseg);
    } else {
      hb_sum<MP>(s8, iv, f, zs + ((uint32_t)st.sg << 8) * kRow, st.nb - q);
    }
    seg_advance(st, ssa, q + 8, nseg);
    if constexpr (FMT == 0) {
      const float sc = e4m3_to_f32_int(lds_u8(sa + ((uint32_t)h >> 1)));
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] = fmaf(s8[m], sc, acc[m]);
    } else {
#pragma unroll
      for (int m = 0; m < MP; ++m) acc[m] += s8[m];
    }
  }
  if (he == h1) {
    finish();
  } else {  // the run ends inside column o: TAIL if it began in the run, else HEAD
    const uint32_t pa = part + (uint32_t)((2 * L + (started ? 1 : 0)) * MP) * 4u;
#pragma unroll
    for (int m = 0; m < MP; ++m) sts_f32(pa + 4u * m, acc[m]);
    if (started) {
      *tail_o = o;
      *tail_he = he;
    }
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
// tile's partial sums in the exchange buffer, then a zero tail of 256 atom rows
// (padding entries read it). Each thread loads a batch of words at once and
// re-reads all of the batch's words that do not yet carry this launch's tag
// together, so a batch costs one round trip to L2 once its writers are done.
template <int MP>
__device__ __forceinline__ void load_ztable(const FusedProj& pp, uint32_t sbase, int tid, uint32_t tag,
                                            volatile int* abort, long long limit) {
  constexpr int NT = kFWarps * 32, B = 8, S = 2;
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
    long long t0 = -1;
    while (true) {
      bool stale = false;
#pragma unroll
      for (int i = 0; i < B; ++i)
#pragma unroll
        for (int s = 0; s < S; ++s) stale |= s < ns[i] && (uint32_t)(v[i][s] >> 32) != tag;
      if (!stale || *abort) break;
      if (t0 < 0) {
        t0 = clock64();
      } else if (clock64() - t0 > limit) {
        atomicOr(&g_dictproj_error, 1u);
        *abort = 1;
        break;
      }
#pragma unroll
      for (int i = 0; i < B; ++i)
#pragma unroll
        for (int s = 0; s < S; ++s)
          if (s < ns[i] && (uint32_t)(v[i][s] >> 32) != tag) v[i][s] = ld_relaxed_u64(pp.zx + s * stride + base + i * NT);
    }
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int e = base + i * NT;
      if (e >= ne) continue;
      float sum = 0.f;
#pragma unroll
      for (int s = 0; s < S; ++s)
        if (s < ns[i]) sum += __uint_as_float((uint32_t)(v[i][s] & 0xffffffffull));
      for (int s = S; s < ns[i]; ++s) {  // tiles split over more than S positions (rare: one read at a time)
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
      constexpr int NT = kFWarps * 32, U = 4;
      const int vpr = pp.ppr * 64, nv = M * vpr;
      for (int v0 = tid; v0 < nv; v0 += U * NT) {  // U loads in flight per thread
        uint4 val[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * NT, m = v / vpr, e = 8 * (v - m * vpr);
          val[u] = v < nv && e < pp.d_in ? ld_cg_v4(pp.X + (size_t)m * pp.d_in + e) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * NT, m = v / vpr, e = 8 * (v - m * vpr);
          if (v < nv)
            sts_u32x4(sbase + pp.xoff + m * prm.xrow + (e >> 8) * 512 + ((e >> 3) & 3) * 128 + ((e >> 5) & 7) * 16,
                      val[u]);
        }
      }
    }
    named_bar_sync(1, kFWarps * 32);
    if (tid == 0) phase_mark(cta, 2);

    // ---- stage 1: partial Z of this CTA's D pieces
    float acc[4][4];
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;
    int cur_tp = -1;
    auto flush = [&](int tp) {
      const uint32_t rb = sbase + prm.red_off + (uint32_t)((tp * kFWarps + warp) * 16 * MP) * 4;
      const int m0 = 2 * tq, m1 = 2 * tq + 1;
      if (m0 < MP) {
        sts_f32(rb + (g * MP + m0) * 4, (acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]));
        sts_f32(rb + ((g + 8) * MP + m0) * 4, (acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2]));
      }
      if (m1 < MP) {
        sts_f32(rb + (g * MP + m1) * 4, (acc[0][1] + acc[1][1]) + (acc[2][1] + acc[3][1]));
        sts_f32(rb + ((g + 8) * MP + m1) * 4, (acc[0][3] + acc[1][3]) + (acc[2][3] + acc[3][3]));
      }
#pragma unroll
      for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;
    };
    unsigned long long s1_wait = 0;  // ns warp 0 waited for dictionary slots (diagnostic)
    for (int j = 0; j < nD; ++j) {
      const int s = j % R;
      unsigned long long tw0 = 0;
      if (tid == 0) asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tw0));
      bool ok = mbar_wait_or_abort(full + s, (uint32_t)((j / R) & 1), s_abort, limit);
      ok = __all_sync(0xffffffffu, ok);
      if (tid == 0) {
        unsigned long long tw1;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tw1));
        s1_wait += tw1 - tw0;
      }
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
    if (prm.zt_resident) {  // (every compute thread calls it: it holds a barrier; an abort only cuts the waits)
      for (int p = 0; p < n; ++p)
        load_ztable<MP>(prm.p[p], sbase, tid, (uint32_t)misc[8 + p], s_abort, limit);
      named_bar_sync(1, kFWarps * 32);
    }
    if (tid == 0) {
      phase_mark(cta, 5);
      if (cta < kPhaseCtas) g_phase[cta * kPhaseSlots + 6] = s1_wait;
    }

    // ---- stage 2: Y = Z C over this CTA's column chunks, in batches of up to W
    // resident chunks of one projection: the batch's half-blocks split evenly over
    // the compute threads, then split columns combined
    constexpr int NL = kFWarps * 32;
    const int W = prm.W;
    int cur_p = -1, nb_done = 0;
    unsigned long long s2_wait = 0;  // ns thread 0 waited for coefficient chunks (diagnostic)
    for (int i0 = 0; i0 < N2; ++nb_done) {
      const int p = desc_p[i0];
      int i1 = i0 + 1;
      while (i1 < N2 && i1 - i0 < W && desc_p[i1] == p) ++i1;
      if (!prm.zt_resident && p != cur_p) {  // one Z table at a time: reload between projections
        named_bar_sync(1, NL);
        load_ztable<MP>(prm.p[p], sbase, tid, (uint32_t)misc[8 + p], s_abort, limit);
        named_bar_sync(1, NL);
      }
      cur_p = p;
      const FusedProj& pp = prm.p[p];
      const int fmt = pp.cfmt, nseg = pp.nseg;
      const uint32_t zs = sbase + pp.zt_off;
      const float yscale = pp.s_C;
      const uint32_t part = sbase + prm.part_off + (uint32_t)(nb_done & 1) * (uint32_t)(2 * NL * MP * 4);
      unsigned long long tw0 = 0;
      if (tid == 0) asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tw0));
      bool ok = true;
      int H = 0;
      for (int i = i0; i < i1; ++i) {
        const int j = nD + i;
        ok = ok && mbar_wait_or_abort(full + j % R, (uint32_t)((j / R) & 1), s_abort, limit);
        H += (int)((desc[i].w - desc[i].z) >> 3);
      }
      if (tid == 0) {
        unsigned long long tw1;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tw1));
        s2_wait += tw1 - tw0;
      }
      ok = ok && !*s_abort;
      const int hq = H / NL, hr = H - hq * NL;
      const int g1 = split_begin(tid + 1, hq, hr);
      int h = split_begin(tid, hq, hr), i = i0, P = 0;
      if (ok && h < g1)
        while (P + (int)((desc[i].w - desc[i].z) >> 3) <= h) P += (int)((desc[i].w - desc[i].z) >> 3), ++i;
      int tail_o = -1, tail_he = 0;  // the column this thread's run ends inside (if it began in the run)
      while (ok && h < g1) {  // the run's part in chunk i (threads step through their parts together)
        const uint4 d = desc[i];
        int to = -1, the = 0;
        const int Hc = (int)((d.w - d.z) >> 3), hi = min(g1 - P, Hc);
        const int s = (nD + i) % R;
        const CChunk c = c_chunk_layout(d.x, d.y, d.z, d.w, (uint32_t)nseg, fmt);
        const uint32_t slot = sbase + (uint32_t)s * kFusedSlotBytes;
        switch (fmt) {  // uniform over the projection
          case 0: stage2_run<MP, 0>(pp, d, c, slot, zs, h - P, hi, tid, part, M, yscale, &to, &the); break;
          case 1: stage2_run<MP, 1>(pp, d, c, slot, zs, h - P, hi, tid, part, M, yscale, &to, &the); break;
          case 2: stage2_run<MP, 2>(pp, d, c, slot, zs, h - P, hi, tid, part, M, yscale, &to, &the); break;
          default: stage2_run<MP, 3>(pp, d, c, slot, zs, h - P, hi, tid, part, M, yscale, &to, &the); break;
        }
        if (to >= 0) {
          tail_o = to;
          tail_he = P + the;
        }
        h = P + hi;
        P += Hc;
        ++i;
      }
      named_bar_sync(1, NL);  // every share of the batch is in `part`
      if (ok && tail_o >= 0 && !*s_abort) {  // TAIL + HEAD of each following thread that starts inside the column
        float y[MP];
        const uint32_t ta = part + (uint32_t)((2 * tid + 1) * MP) * 4u;
#pragma unroll
        for (int m = 0; m < MP; ++m) y[m] = lds_f32(ta + 4u * m);
        for (int Lx = tid + 1; Lx < NL && split_begin(Lx, hq, hr) < tail_he; ++Lx) {
          const uint32_t ha = part + (uint32_t)(2 * Lx * MP) * 4u;
#pragma unroll
          for (int m = 0; m < MP; ++m) y[m] += lds_f32(ha + 4u * m);
        }
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < M) pp.Y[(size_t)m * pp.d_out + tail_o] = __float2half_rn(y[m] * yscale);
      }
      for (i = i0; i < i1; ++i) {  // empty columns are zero; then release each chunk's slot
        const uint4 d = desc[i];
        const int s = (nD + i) % R;
        if (ok && !*s_abort) {
          const CChunk c = c_chunk_layout(d.x, d.y, d.z, d.w, (uint32_t)nseg, fmt);
          const uint32_t cpa = sbase + (uint32_t)s * kFusedSlotBytes + c.cp_dst - c.cp_src;
          for (int o = (int)d.x + tid; o < (int)d.y; o += NL)
            if (lds_u32(cpa + 4u * (uint32_t)o) == lds_u32(cpa + 4u * (uint32_t)o + 4u))
              for (int m = 0; m < M; ++m) pp.Y[(size_t)m * pp.d_out + o] = __float2half_rn(0.f);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(empty + s);
      }
      i0 = i1;
    }
    if (tid == 0 && cta < kPhaseCtas) {
      phase_mark(cta, 13);
      g_phase[cta * kPhaseSlots + 12] = s2_wait;
      g_phase[cta * kPhaseSlots + 14] = (unsigned long long)N2;
      g_phase[cta * kPhaseSlots + 15] = (unsigned long long)nD;
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
  const int part = 2 * 2 * kFWarps * 32 * mp * 4;  // stage-2 partial sums, two buffers
  auto batch_of = [](int R) { return std::max(1, std::min(kMaxStage2Batch, R - 2)); };
  auto total = [&](int R, int U) { return 1024 + R * kFusedSlotBytes + U + part + fused_ctl_bytes(R); };
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
  pl.part_off = pl.R * kFusedSlotBytes + pl.U;
  pl.W = batch_of(pl.R);
  pl.bar_off = pl.part_off + part;
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
  prm.part_off = pl.part_off;
  prm.W = pl.W;
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

// Self-test of this file's bounded-wait error path (its own device error word):
// one warp waits on an mbarrier that expects two arrivals and receives one, so
// the wait can only end by its limit of `cycles` SM clocks. Nothing else is in
// flight when it gives up.
__global__ void k_wait_probe_fused(long long cycles) {
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

cudaError_t launch_wait_probe_fused(long long cycles, cudaStream_t stream) {
  k_wait_probe_fused<<<1, 32, 0, stream>>>(cycles);
  return cudaGetLastError();
}

cudaError_t take_fused_error(unsigned int* out) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_dictproj_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_dictproj_error, &zero, sizeof(unsigned int));
}

}  // namespace dictproj
