// Prefill path (M > 8 tokens): both stages of Y = (X·D_g)·C_l as tcgen05 GEMMs.
//
// At prefill the dictionary stage Z = X·D_g is a dense contraction with about
// 2·M·d_in·k flops on d_in·k·9/16 bytes of packed dictionary, far above the
// HBM ridge, so it runs on the 5th-generation tensor cores (DictLLM technical
// review, Eq. (1) and "Efficiency" section; the compressed factors replace one
// d_in x d_out product by a d_in x k product and a sparse k x d_out one).
//
//   k_dict_prefill   Z[M][k] = s_D · X[M][d_in] · D^[d_in][k], as Z^T tiles of
//       128 atoms x nt tokens: the packed E2M1 codes and the X tile arrive by
//       TMA; sixteen producer warps decode the codes (E2M1 x E4M3 block scale,
//       exact in fp16) straight into tensor memory as operand A; one thread
//       issues tcgen05.mma with B = X in shared memory and the fp32 accumulator
//       in tensor memory. The epilogue applies s_D in fp32 before rounding Z to
//       fp16 (the unscaled sum can exceed the fp16 range). For few tokens the
//       d_in stages of a tile are split over a thread-block cluster and summed
//       over distributed shared memory.
//   k_densify_coeff  Cd[d_out][k] = C^ (fp16, zeros off the support)
//   k_gemm_tma       Y[M][d_out] = s_C · Z[M][k] · Cd^T, both operands by TMA.
//       At prefill the tensor cores run the zeros of C faster than CUDA cores run
//       only its nonzeros (dense fp16 rate / fp32 FMA rate >> 1/rho).
//
// Every spin-wait is bounded; a wait that gives up sets bit 0 of the device
// error word and the kernel unwinds (frees its tensor memory) without hanging.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "dictproj_internal.h"
#include "kernels.h"

namespace dictproj {
namespace {

constexpr int BM = 128;                 // tokens per tile (MMA M, tensor-memory lanes)
constexpr int BN = 256;                 // atoms / output columns per tile (MMA N)
constexpr int BK = 64;                  // reduction elements per stage (one 128-byte swizzle row)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int B_BYTES = BN * BK * 2;    // 32 KB
constexpr int kTA = 128;                // atoms per dictionary-stage tile (MMA M)
constexpr int kGemmThreads = 320;       // warp 0 TMA, warp 1 MMA + TMEM, warps 2..9 producers/epilogue
constexpr int kProducerWarps = 8;
constexpr int kTmemCols = 256;          // fp32 accumulator: 128 lanes x 256 columns
constexpr int kScaleAhead = 4;          // block-scale look-ahead, in stages of one producer group

constexpr size_t kGemmSmem = (size_t)STAGES * (A_BYTES + B_BYTES) + 1024 + 256;

// ---- tcgen05 / TMA primitives ------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// Thread-block cluster: barrier over all threads of all CTAs, and loads from
// another CTA's shared memory (distributed shared memory).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_dsmem(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_v4f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}
// D (tensor memory) (+)= A (shared memory) x B (shared memory)
__device__ __forceinline__ void mma_f16_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D (tensor memory) (+)= A (tensor memory: lane = row, two fp16 per column) x B (shared memory)
__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane; waits for completion.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// 32 consecutive fp32 accumulator columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void sts_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}


// One 128 x 256 output tile of out = scale · A · B^T with A (M x K) and B
// (N x K) fp16 K-major, both brought by TMA with 128-byte swizzle; one thread
// issues tcgen05.mma (M=128, N=256, K=16) into a fp32 accumulator in tensor
// memory; eight warps run the epilogue.
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_tma(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, int M, int N,
               int K, int bn, float scale, __half* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled operand tiles must start on 1024-byte shared-memory boundaries
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sa = smem;
  uint8_t* sb = sa + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sb + STAGES * B_BYTES);
  uint64_t* full = bars;               // TMA bytes of the stage landed
  uint64_t* empty = bars + STAGES;     // MMAs of the stage completed
  uint64_t* accf = bars + 2 * STAGES;  // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * bn, m0 = blockIdx.y * BM;
  const int nk = (K + BK - 1) / BK;
  // kind::f16, A and B fp16, D fp32, K-major, M = 128, N = bn
  const uint32_t idesc = (1u << 4) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // A and B may be the previous kernels' output; nothing below reads or writes
  // global memory before this point.
  grid_dependency_wait();

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      for (int s = 0; s < nk; ++s) {
        const int slot = s % STAGES, round = s / STAGES;
        if (s >= STAGES && !mbar_wait_bounded(&empty[slot], (round - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[slot], A_BYTES + bn * BK * 2);
        tma_load_2d(smem_u32(sa + slot * A_BYTES), &tm_a, s * BK, m0, &full[slot]);
        tma_load_2d(smem_u32(sb + slot * B_BYTES), &tm_b, s * BK, n0, &full[slot]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int s = 0; s < nk; ++s) {
        const int slot = s % STAGES, round = s / STAGES;
        if (!mbar_wait_bounded(&full[slot], round & 1)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(sa + slot * A_BYTES), b = smem_u32(sb + slot * B_BYTES);
#pragma unroll
        for (int j = 0; j < BK / 16; ++j)
          mma_f16_ss(tmem, smem_desc_sw128(a + 32 * j), smem_desc_sw128(b + 32 * j), idesc, (s | j) != 0);
        mma_commit(&empty[slot]);
      }
      mma_commit(accf);
    }
  } else {
    // Epilogue: warp w reads tensor-memory lanes 32·(w % 4) .. +31 (its tokens)
    // and every other 32-column chunk of the bn accumulator columns.
    const int q = warp & 3, half = (warp - 2) >> 2;
    const bool ok = mbar_wait_bounded(accf, 0);
    tc_fence_after();
    const int row = m0 + 32 * q + lane;
    const bool vec = (N & 7) == 0;
    const int nlim = min(N, n0 + bn);
#pragma unroll 1
    for (int c = half; 32 * c < bn; c += 2) {
      const int col = 32 * c;
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + col, v);
      if (!ok || row >= M) continue;
      __half* orow = out + (size_t)row * N;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gc = n0 + col + 8 * j;
        if (gc >= nlim) break;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * j + e]) * scale;
        if (vec) {
          uint4 o;
          o.x = pack_h2(f[0], f[1]);
          o.y = pack_h2(f[2], f[3]);
          o.z = pack_h2(f[4], f[5]);
          o.w = pack_h2(f[6], f[7]);
          *reinterpret_cast<uint4*>(orow + gc) = o;
        } else {
          for (int e = 0; e < 8 && gc + e < nlim; ++e) orow[gc + e] = __float2half_rn(f[e]);
        }
      }
    }
  }
  __syncwarp();
  trigger_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- dictionary stage: Z^T tile = D^T tile (tensor memory) x X tile (shared memory) -------------
// The 128 atoms of a tile are the MMA's M rows: producer warps decode their
// NVFP4 codes into fp16 and store them straight into tensor memory (operand A
// of tcgen05.mma .kind::f16 with A in tensor memory), so the decoded
// dictionary never passes through shared memory; only X (operand B, nt tokens
// x 64) and the packed codes do. The accumulator holds Z^T (atoms x tokens).
// The token-tile width nt (a multiple of 16, at most 256) is chosen per call so
// that the tiles fill whole waves of the GPU.
struct DictTile {
  // Two producer groups of 8 warps take alternate stages, so that the latency of
  // one stage's decode (shared-memory load, conversion, tensor-memory store and
  // its wait) overlaps the next one's.
  static constexpr int kGroups = 2;
  static constexpr int kThreads = 64 + 32 * 8 * kGroups;
  static constexpr int kMaxN = 256;
  static constexpr int kStages = 6;
  static constexpr int kXBytes = kMaxN * BK * 2;    // X tile slot: up to 256 tokens x 64 fp16
  static constexpr int kRawBytes = kTA * BK / 2;    // codes: 128 atoms x 32 bytes
  static constexpr int kAcol = kMaxN;               // first tensor-memory column of the A ring
  static constexpr int kCols = 512;                 // accumulator + 32 per stage, rounded up
  static_assert(kMaxN + 32 * kStages <= kCols, "tensor memory");
  static constexpr size_t smem = (size_t)kStages * (kXBytes + kRawBytes) + 1024 + 256;
};

// Split-K (small M): with gridDim.z = S > 1 the S CTAs of a cluster (1, 1, S)
// take consecutive ranges of the d_in stages of one (atom tile, token tile);
// each leaves its fp32 partial tile in its own shared memory, and CTA r of the
// cluster sums the S partials of its share of the token columns in rank order
// over distributed shared memory (deterministic), applies s_D and writes Z.
__global__ void __launch_bounds__(DictTile::kThreads, 1)
    k_dict_prefill(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
                   const uint8_t* __restrict__ scales, int M, int k, int d_in, int nt, float s_D,
                   __half* __restrict__ Z) {
  using T = DictTile;
  constexpr int S = T::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sx = smem;
  uint8_t* sr = sx + S * T::kXBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sr + S * T::kRawBytes);
  uint64_t* full = bars;           // X tile and codes of the stage landed
  uint64_t* afull = bars + S;      // producers stored the decoded A slice in tensor memory
  uint64_t* empty = bars + 2 * S;  // MMAs of the stage completed
  uint64_t* accf = bars + 3 * S;   // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a0 = blockIdx.x * kTA, m0 = blockIdx.y * nt;
  const int nsplit = (int)gridDim.z, split = (int)blockIdx.z;
  const int nk_all = (d_in + BK - 1) / BK;
  const int s_lo = (int)((long)nk_all * split / nsplit);  // this CTA's stages [s_lo, s_lo + nk)
  const int nk = (int)((long)nk_all * (split + 1) / nsplit) - s_lo;
  // kind::f16, A and B fp16, D fp32, K-major, M = 128 atoms, N = nt tokens
  const uint32_t idesc = (1u << 4) | ((uint32_t)(nt >> 3) << 17) | ((uint32_t)(kTA >> 4) << 24);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], kProducerWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, T::kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();  // X may be the previous kernel's output

  if (warp == 0) {
    if (lane == 0) {  // TMA producer: X tile and packed codes per stage
      for (int s = 0; s < nk; ++s) {
        const int slot = s % S, round = s / S;
        if (s >= S && !mbar_wait_bounded(&empty[slot], (round - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[slot], nt * BK * 2 + T::kRawBytes);
        tma_load_2d(smem_u32(sx + slot * T::kXBytes), &tm_x, (s_lo + s) * BK, m0, &full[slot]);
        tma_load_2d(smem_u32(sr + slot * T::kRawBytes), &tm_codes, (s_lo + s) * (BK / 2), a0, &full[slot]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int s = 0; s < nk; ++s) {
        const int slot = s % S, round = s / S;
        if (!mbar_wait_bounded(&full[slot], round & 1)) break;
        if (!mbar_wait_bounded(&afull[slot], round & 1)) break;
        tc_fence_after();
        const uint32_t x = smem_u32(sx + slot * T::kXBytes);
        const uint32_t a = tmem + T::kAcol + 32 * slot;
#pragma unroll
        for (int j = 0; j < BK / 16; ++j) mma_f16_ts(tmem, a + 8 * j, smem_desc_sw128(x + 32 * j), idesc, (s | j) != 0);
        mma_commit(&empty[slot]);
      }
      mma_commit(accf);
    }
  } else {
    // Warp w owns tensor-memory lanes 32·(w % 4) .. +31 (atoms a0 + that), half
    // h of each stage's 64 reduction elements, and the stages s = g (mod groups).
    const int e = warp - 2, g = e >> 3;
    const int q = warp & 3, h = (e >> 2) & 1;
    const int r = 32 * q + lane;
    const bool row_ok = a0 + r < k;
    const int nblk = d_in / 16;  // even
    const uint8_t* srow = scales + (size_t)(row_ok ? a0 + r : 0) * nblk + 2 * h;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // Two E4M3 block scales per stage (blocks 4s + 2h, +1) travel in a register
    // ring loaded kScaleAhead of this group's stages ahead of use. The ring is
    // indexed statically (the loop over it is unrolled): moving a register whose
    // load is still in flight would wait for that load.
    constexpr int G = T::kGroups, R = kScaleAhead;
    auto scale_at = [&](int st) -> uint32_t {  // st: this CTA's stage number
      return (row_ok && st < nk && 4 * (s_lo + st) + 2 * h < nblk) ? ld_stream_u16(srow + 4 * (s_lo + st)) : 0u;
    };
    uint32_t scr[R];
#pragma unroll
    for (int i = 0; i < R; ++i) scr[i] = scale_at(g + G * i);
    bool live = true;
    for (int base = g; live && base < nk; base += G * R) {
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int s = base + G * i;
        if (!live || s >= nk) break;
        const int slot = s % S, round = s / S;
        const uint32_t sc = scr[i];
        scr[i] = scale_at(s + G * R);
        if (!mbar_wait_bounded(&full[slot], round & 1)) {
          live = false;
          break;
        }
        const uint4 c = lds_u32x4(smem_u32(sr + slot * T::kRawBytes) + r * 32 + 16 * h);
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        const uint32_t hs = e4m3x2_to_f16x2(sc);
        const uint32_t scl[2] = {dup_lo(hs), dup_hi(hs)};
        uint32_t o[16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t f[4];
          e2m1x8_to_f16x2x4(w[cc], f);
#pragma unroll
          for (int t = 0; t < 4; ++t) o[4 * cc + t] = hmul2_u32(f[t], scl[cc >> 1]);
        }
        tmem_st16(tmem + lane_base + T::kAcol + 32 * slot + 16 * h, o);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[slot]);
      }
    }
    // Epilogue: Z[m][a0 + r]; the 32-token column chunks of the accumulator go
    // round-robin to the 2·groups warps of each lane quadrant.
    const bool ok = mbar_wait_bounded(accf, 0);
    tc_fence_after();
    const int lim = min(nt, M - m0);  // valid token columns of this tile
    // split-K: the partial tile goes to this CTA's shared memory, token-major
    // (the stage buffers are idle once the accumulator is complete)
    float* part = reinterpret_cast<float*>(smem);
#pragma unroll 1
    for (int c = e >> 2; 32 * c < nt; c += 2 * G) {
      const int col = 32 * c;
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + col, v);
      if (nsplit > 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) part[(col + j) * kTA + r] = ok ? __uint_as_float(v[j]) : 0.f;
        continue;
      }
      if (!ok || !row_ok) continue;
      __half* zc = Z + (size_t)(m0 + col) * k + a0 + r;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col + j < lim) zc[(size_t)j * k] = __float2half_rn(__uint_as_float(v[j]) * s_D);
    }
  }
  __syncwarp();
  trigger_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::kCols);
  }
  if (nsplit > 1) {
    // every partial is in place: CTA `split` sums its token columns over the
    // cluster's CTAs in rank order, four atoms per thread
    cluster_sync_all();
    const int lim = min(nt, M - m0);
    const int c_lo = (int)((long)nt * split / nsplit), c_hi = (int)((long)nt * (split + 1) / nsplit);
    const uint32_t pbase = smem_u32(smem);
    for (int i = threadIdx.x; i < (c_hi - c_lo) * (kTA / 4); i += blockDim.x) {
      const int col = c_lo + i / (kTA / 4), a4 = 4 * (i % (kTA / 4));
      const uint32_t off = (uint32_t)(col * kTA + a4) * 4u;
      float4 acc = ld_dsmem_v4f(map_dsmem(pbase + off, 0));
      for (int rk = 1; rk < nsplit; ++rk) {
        const float4 q = ld_dsmem_v4f(map_dsmem(pbase + off, (uint32_t)rk));
        acc.x += q.x;
        acc.y += q.y;
        acc.z += q.z;
        acc.w += q.w;
      }
      if (col < lim && a0 + a4 < k) {  // k % 16 == 0: the four atoms are all in range
        __half2* zc = reinterpret_cast<__half2*>(Z + (size_t)(m0 + col) * k + a0 + a4);
        zc[0] = __floats2half2_rn(acc.x * s_D, acc.y * s_D);
        zc[1] = __floats2half2_rn(acc.z * s_D, acc.w * s_D);
      }
    }
    cluster_sync_all();  // no CTA leaves while another still reads its partial tile
  }
}

// Dense fp16 copy of C^ (atom-major rows per output column: Cd[o][a]), zeros off
// the support. One warp per column builds the row in shared memory, then writes
// it out with 16-byte stores. A lane takes 4 consecutive stored entries per
// 128-entry chunk (one 4-byte index load, one 2-byte code load, one scale byte:
// columns are padded to multiples of 16 entries, so the loads are aligned), and
// the next chunk's loads are issued before the current one is scattered.
// Entries with code 0 (value 0, and the padding at the end of each column) are
// skipped. The column's segment starts sit in shared memory.
// Four consecutive stored values (entry e, e % 4 == 0) in format FMT: raw code
// bits (NVFP4: 4 nibbles, FP8 / INT8: 4 bytes, FP16: 4 halves) and, for NVFP4,
// the block's E4M3 scale byte.
template <int FMT>
__device__ __forceinline__ uint2 load4_values(const uint8_t* codes, uint32_t e) {
  if constexpr (FMT == 0) return make_uint2(*reinterpret_cast<const uint16_t*>(codes + (e >> 1)), 0u);
  else if constexpr (FMT == 1) return *reinterpret_cast<const uint2*>(codes + 2 * e);
  else return make_uint2(*reinterpret_cast<const uint32_t*>(codes + e), 0u);
}
// fp16 value of entry t (0..3) of a group loaded by load4_values (unscaled by s_C;
// NVFP4: E2M1 x E4M3 block scale, exact in fp16), and whether it is zero.
template <int FMT>
__device__ __forceinline__ uint32_t value4(uint2 v, uint32_t sv, int t) {
  if constexpr (FMT == 0) {
    const uint32_t code = (v.x >> (4 * t)) & 15;
    return (code & 7) == 0 ? 0u : hmul2_u32(e2m1x2_to_f16x2(code), sv) & 0xFFFF;
  } else if constexpr (FMT == 1) {
    return ((t < 2 ? v.x : v.y) >> (16 * (t & 1))) & 0xFFFF;
  } else if constexpr (FMT == 2) {
    const uint32_t b = (v.x >> (8 * t)) & 0xFF;
    return (b & 0x7F) == 0 ? 0u : e4m3x2_to_f16x2(b) & 0xFFFF;
  } else {
    const int c = (int)(int8_t)((v.x >> (8 * t)) & 0xFF);
    return (uint32_t)__half_as_ushort(__int2half_rn(c));
  }
}

template <int FMT>
__global__ void __launch_bounds__(256)
    k_densify_coeff(const uint32_t* __restrict__ col_ptr, const uint8_t* __restrict__ codes,
                    const uint8_t* __restrict__ scales, const uint8_t* __restrict__ idx,
                    const uint16_t* __restrict__ seg_start, int k, int d_out, int nseg, __half* __restrict__ cd) {
  extern __shared__ __align__(16) uint8_t dsm[];
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * nw + warp;
  grid_dependency_wait();  // Cd may still be read by the previous coefficient GEMM
  if (o >= d_out) return;
  __half* row = reinterpret_cast<__half*>(dsm) + (size_t)warp * k;
  uint16_t* ss = reinterpret_cast<uint16_t*>(dsm + (size_t)nw * k * 2) + (size_t)warp * nseg;
  const uint32_t rbase = smem_u32(row);
  for (int c = lane; c < k / 8; c += 32) sts_v4(rbase + 16 * c, 0, 0, 0, 0);
  for (int j = lane; j < nseg; j += 32) ss[j] = seg_start[(size_t)o * nseg + j];
  __syncwarp();
  const uint32_t e0 = col_ptr[o], e1 = col_ptr[o + 1];
  int seg = 0;  // segment of this lane's entries; they only increase
  uint32_t i4 = 0, sc = 0;
  uint2 c4 = make_uint2(0, 0);
  {
    const uint32_t e = e0 + 4 * lane;
    if (e < e1) {
      i4 = *reinterpret_cast<const uint32_t*>(idx + e);
      c4 = load4_values<FMT>(codes, e);
      if (FMT == 0) sc = scales[e >> 4];
    }
  }
  for (uint32_t base = e0; base < e1; base += 128) {
    const uint32_t e = base + 4 * lane, en = e + 128;
    uint32_t ni4 = 0, nsc = 0;  // next chunk, loaded before this one is scattered
    uint2 nc4 = make_uint2(0, 0);
    if (en < e1) {
      ni4 = *reinterpret_cast<const uint32_t*>(idx + en);
      nc4 = load4_values<FMT>(codes, en);
      if (FMT == 0) nsc = scales[en >> 4];
    }
    if (e < e1) {
      const uint32_t sv = FMT == 0 ? dup_lo(e4m3x2_to_f16x2(sc)) : 0u;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t h = value4<FMT>(c4, sv, t);
        if ((h & 0x7FFF) == 0) continue;  // +-0 and padding
        const int q = (int)(e - e0) + t;
        while (seg + 1 < nseg && (int)ss[seg + 1] <= q) ++seg;
        const uint32_t atom = 256u * seg + ((i4 >> (8 * t)) & 255);
        row[atom] = __ushort_as_half((unsigned short)h);
      }
    }
    i4 = ni4;
    c4 = nc4;
    sc = nsc;
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(cd + (size_t)o * k);
  for (int c = lane; c < k / 8; c += 32) dst[c] = lds_u32x4(rbase + 16 * c);
}

// ---- host side ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static std::mutex g_enc_mu;
static EncodeTiledFn g_encode = nullptr;

static cudaError_t get_encoder(EncodeTiledFn* fn) {
  std::lock_guard<std::mutex> lk(g_enc_mu);
  if (!g_encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = g_encode;
  return cudaSuccess;
}

}  // namespace

// 2-D row-major map: rows x inner elements, row stride in bytes, box inner x rows.
cudaError_t encode_tiled_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
                             uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                             CUtensorMapSwizzle swz) {
  EncodeTiledFn enc;
  cudaError_t e = get_encoder(&enc);
  if (e != cudaSuccess) return e;
  const cuuint64_t gdim[2] = {inner, rows};
  const cuuint64_t gstride[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, type, 2, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {
static cudaError_t encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
                             uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                             CUtensorMapSwizzle swz) {
  return encode_tiled_2d(map, type, base, inner, rows, row_bytes, box_inner, box_rows, swz);
}

static cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

}  // namespace

cudaError_t prepare_prefill_kernels(int device) {
  (void)device;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_gemm_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem)) ||
      (e = cudaFuncSetAttribute(k_dict_prefill, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)DictTile::smem)))
    return e;
  if ((e = cudaFuncSetAttribute(k_densify_coeff<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024)) ||
      (e = cudaFuncSetAttribute(k_densify_coeff<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024)) ||
      (e = cudaFuncSetAttribute(k_densify_coeff<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024)))
    return e;
  return cudaFuncSetAttribute(k_densify_coeff<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

// Self-test of this file's bounded-wait error path (its own device error word):
// one warp waits on an mbarrier that expects two arrivals and receives one, so
// the wait can only end by its limit of `cycles` SM clocks. Nothing else is in
// flight when it gives up.
__global__ void k_wait_probe_prefill(long long cycles) {
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

cudaError_t launch_wait_probe_prefill(long long cycles, cudaStream_t stream) {
  k_wait_probe_prefill<<<1, 32, 0, stream>>>(cycles);
  return cudaGetLastError();
}

cudaError_t take_prefill_error(unsigned int* out) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_dictproj_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_dictproj_error, &zero, sizeof(unsigned int));
}

cudaError_t encode_dict_codes_map(const dictproj_group* g, CUtensorMap* map) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, g->codes, (uint64_t)g->d_in / 2, (uint64_t)g->k,
                   (uint64_t)g->d_in / 2, BK / 2, kTA, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Width w (a multiple of 16, at most 256) of the tiles that split `extent`
// elements, with `other` tiles along the other side: fewest padded columns per SM
// over the waves the grid takes, counting each tile's fixed per-stage cost as 32
// columns.
int prefill_tile_width(long extent, long other, int n_sm) {
  int best = 256;
  double best_cost = 1e300;
  for (long t = (extent + 255) / 256; t <= (extent + 15) / 16; ++t) {
    const long w = ((extent + t - 1) / t + 15) / 16 * 16;
    const long tiles = other * ((extent + w - 1) / w);
    const long waves = (tiles + n_sm - 1) / n_sm;
    const double cost = (double)waves * (double)(w + 32);
    if (cost < best_cost) {
      best_cost = cost;
      best = (int)w;
    }
  }
  return best;
}

// Clusters of S CTAs of the prefill dictionary kernel (one CTA per SM at its
// shared memory) that the device holds at once, from the occupancy query;
// cached per device and S.
static int dict_clusters_that_fit(int S) {
  static std::atomic<int> cache[16][9];
  static std::once_flag once;
  std::call_once(once, [] {
    for (auto& d : cache)
      for (auto& c : d) c.store(-1);
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16 || S < 1 || S > 8) return 0;
  int v = cache[dev][S].load();
  if (v >= 0) return v;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, S);
  cfg.blockDim = dim3(DictTile::kThreads);
  cfg.dynamicSmemBytes = DictTile::smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)S;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)k_dict_prefill, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[dev][S].store(n);
  return n;
}

PrefillDictPlan prefill_dict_plan(int M, int d_in, int k, int n_sm) {
  PrefillDictPlan p;
  const int tiles_a = (k + kTA - 1) / kTA, nk = (d_in + BK - 1) / BK;
  p.nt = prefill_tile_width(M, tiles_a, n_sm);
  p.splits = 1;
  if (M <= 2 * DictTile::kMaxN) {
    // Few tokens: the d_in stages split over a cluster of up to 8 CTAs (each at
    // least 4 stages), so that the grid fills the GPU without every token tile
    // decoding the same dictionary tile again. Of the splits whose clusters are
    // all resident at once, the one with the most CTAs; ties go to fewer token
    // tiles (less decoding).
    int best = 0;
    for (int tm = (M + DictTile::kMaxN - 1) / DictTile::kMaxN; tm <= 4; tm *= 2) {
      const int nt = ((M + tm - 1) / tm + 15) / 16 * 16;
      if (nt < 16 || (M + nt - 1) / nt != tm) break;
      const int tiles = tiles_a * tm;
      for (int S = std::min({8, n_sm / tiles, nk / 4}); S >= 2; --S)
        if (dict_clusters_that_fit(S) >= tiles) {
          if (tiles * S > best) {
            best = tiles * S;
            p.nt = nt;
            p.splits = S;
          }
          break;
        }
    }
  }
  return p;
}

cudaError_t launch_dict_prefill(const dictproj_group* g, const __half* X, int M, __half* Z, cudaStream_t stream) {
  const PrefillDictPlan plan = prefill_dict_plan(M, g->d_in, g->k, g->n_sm);
  int nt = plan.nt;
  CUtensorMap tx;
  cudaError_t e = encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, (uint64_t)g->d_in, (uint64_t)M,
                            (uint64_t)g->d_in * 2, BK, nt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((g->k + kTA - 1) / kTA, (M + nt - 1) / nt, plan.splits);
  cfg.blockDim = dim3(DictTile::kThreads);
  cfg.dynamicSmemBytes = DictTile::smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2] = {pdl_attr(), {}};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (plan.splits > 1) {  // the split CTAs of a tile form one cluster
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = (unsigned)plan.splits;
    cfg.numAttrs = 2;
  }
  const uint8_t* sc = g->scales;
  int k = g->k, d_in = g->d_in;
  float s = g->s;
  void* args[] = {(void*)&tx, (void*)&g->codes_map, (void*)&sc, &M, &k, &d_in, &nt, &s, (void*)&Z};
  return cudaLaunchKernelExC(&cfg, (const void*)k_dict_prefill, args);
}

cudaError_t launch_densify_coeff(const dictproj_layer* l, __half* Cd, cudaStream_t stream) {
  if (l->ifmt != DICTPROJ_IFMT_U8) return launch_densify_index(l, Cd, stream);
  const size_t per_warp = (size_t)l->k * 2 + (size_t)l->nseg * 2;
  const int warps = std::max(1, std::min(8, (int)((200 * 1024) / per_warp)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((l->d_out + warps - 1) / warps);
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = (size_t)warps * per_warp;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int k = l->k, d_out = l->d_out, nseg = l->nseg;
  void* args[] = {(void*)&l->col_ptr, (void*)&l->codes, (void*)&l->scales, (void*)&l->idx, (void*)&l->seg_start,
                  &k, &d_out, &nseg, (void*)&Cd};
  switch (l->cfmt) {
    case 0: return cudaLaunchKernelExC(&cfg, (const void*)k_densify_coeff<0>, args);
    case 1: return cudaLaunchKernelExC(&cfg, (const void*)k_densify_coeff<1>, args);
    case 2: return cudaLaunchKernelExC(&cfg, (const void*)k_densify_coeff<2>, args);
    default: return cudaLaunchKernelExC(&cfg, (const void*)k_densify_coeff<3>, args);
  }
}

cudaError_t launch_coeff_prefill(const dictproj_layer* l, const __half* Z, const __half* Cd, int M, __half* Y,
                                 cudaStream_t stream) {
  CUtensorMap ta, tb;
  cudaError_t e = encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Z, (uint64_t)l->k, (uint64_t)M,
                            (uint64_t)l->k * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  int bn = prefill_tile_width(l->d_out, (M + BM - 1) / BM, l->n_sm);
  e = encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Cd, (uint64_t)l->k, (uint64_t)l->d_out, (uint64_t)l->k * 2, BK,
                bn, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((l->d_out + bn - 1) / bn, (M + BM - 1) / BM);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int N = l->d_out, K = l->k;
  float s = l->s;
  void* args[] = {(void*)&ta, (void*)&tb, &M, &N, &K, &bn, &s, (void*)&Y};
  return cudaLaunchKernelExC(&cfg, (const void*)k_gemm_tma, args);
}

}  // namespace dictproj
