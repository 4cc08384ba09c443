// Kernel launchers (host side), one per stage and path.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <vector>

#include "dictproj_internal.h"

namespace dictproj {

// decode path (M <= 8): Z fp32 [k][mp], mp = next power of two >= M (at most 8),
// written by the dictionary stage as `slices` partial sums Zpart[slice][k][mp]
int decode_mp(int M);
cudaError_t prepare_decode_kernels(int device);

struct DictPlan {
  int J;       // 128-element units per warp
  int slices;  // d_in slices = grid.y
};
DictPlan dict_plan(int d_in, int k, int n_sm, int M, bool one_slice);
// One plan for a batched launch: a common J, chosen by a fitted cost (waves x
// (fixed + rows per CTA)), so CTAs per projection follow its dictionary bytes;
// never more slices than J = 1 gives (dict_max_slices, the group's Z scratch).
void dict_plan_batch(int n, const int* d_in, const int* k, int n_sm, int M, DictPlan* plans);
// CTAs of a batched gather launch per projection (n_sm in all, at least one
// each), given each projection's stored entries and columns: handed out so that
// the projection that would finish last gets the next one (a fitted cost per
// column and per 256-entry window, whole columns per warp).
void gather_batch_shares(int n, const size_t* entries, const int* columns, int n_sm, int* share);
int dict_max_slices(int d_in, int k, int n_sm);  // over all decode M
cudaError_t launch_dict_decode(const dictproj_group* g, const __half* X, int M, int mp, float* Zpart,
                               const DictPlan& plan, cudaStream_t stream);
cudaError_t launch_coeff_decode(const dictproj_layer* l, const float* Zpart, int nslices, int M, int mp,
                                __half* Y, cudaStream_t stream);
// Batches of up to 4 independent projections in one launch per stage.
constexpr int kDecodeMaxBatch = 4;
cudaError_t launch_dict_decode_batch(int n, const dictproj_group* const* g, const __half* const* X, int M,
                                     int mp, float* const* Zpart, const DictPlan* plans, cudaStream_t stream);
cudaError_t launch_coeff_decode_batch(int n, const dictproj_layer* const* l, const float* const* Zpart,
                                      const int* nslices, int M, int mp, __half* const* Y, cudaStream_t stream);
// Whether one gather launch serves the batch's coefficient stage.
bool decode_batch_gathers(int n, const dictproj_layer* const* l);

// Whether the gather kernel serves a layer (every column <= 1280 padded
// entries, at most 32 segments); other layers use the direct kernel.
bool gather_supported(const uint32_t* pcol_ptr, int d_out, int nseg);
// Whether the coefficient kernels' shared memory, (k + 256) * mp floats of Z,
// fits the device's per-block limit.
bool coeff_smem_fits(int k, int mp, int device);
// One warp whose bounded wait can only end by its limit (error-path self-test).
cudaError_t launch_wait_probe(long long cycles, cudaStream_t stream);
// The same probe in the prefill and fused kernel files (each file has its own
// device error word).
cudaError_t launch_wait_probe_prefill(long long cycles, cudaStream_t stream);
cudaError_t launch_wait_probe_fused(long long cycles, cudaStream_t stream);
// Read and clear the device error word of the decode kernels.
cudaError_t take_decode_error(unsigned int* out);
// Diagnostic timestamps of the gather kernel (buf null: off).
cudaError_t set_gather_times(unsigned long long* buf, int max_ctas);
cudaError_t take_fused_error(unsigned int* out);

// fused decode path (M <= 8): one kernel per call, both stages, weights staged
// through shared memory by TMA (fused.cu)
constexpr int kFusedSlotBytes = 16384;  // one ring slot
struct FusedLaunchPlan {
  int mp, R, U, smem, zt_resident, stage_x, xrow, red_off, bar_off, part_off, W, n_tp;
  int xoff[4], xfirst[4], xslot[4], zt_off[4];
};
cudaError_t prepare_fused_kernels(int device);
// Bitmap and block-structured C_l (indexfmt.cu)
cudaError_t prepare_index_kernels(int device);
bool index_smem_fits(int k, int mp, int device);
cudaError_t launch_coeff_index(const dictproj_layer* l, const float* Zpart, int nslices, int M, int mp, __half* Y,
                               cudaStream_t stream);
cudaError_t launch_densify_index(const dictproj_layer* l, __half* Cd, cudaStream_t stream);
// Tile-major dictionary copy (from the host's packed arrays), exchange buffer and
// ticket of a group (sets g->fused_ok when the shape is served; allocation
// failures are returned).
cudaError_t fused_group_setup(dictproj_group* g, const uint8_t* codes, const uint8_t* scales, bool* ok);
// Column chunks of a layer for G positions: off[G+1] into chunks {o_a, o_b, E_a, E_b}.
// False if a column does not fit a ring slot (the layer then runs the two-kernel path).
bool fused_layer_plan(const uint32_t* pcol_ptr, int d_out, int nseg, int fmt, int G, std::vector<uint32_t>& off,
                      std::vector<uint4>& chunks, int* max_per_pos);
// Shared-memory plan of one launch; false if the fused kernel does not serve it.
bool fused_plan_launch(int n, const dictproj_group* const* g, const dictproj_layer* const* l,
                       const __half* const* X, int M, int smem_optin, FusedLaunchPlan* out);
cudaError_t launch_fused(int n, const dictproj_group* const* g, const dictproj_layer* const* l,
                         const __half* const* X, __half* const* Y, int M, const FusedLaunchPlan& pl,
                         long long wait_limit, cudaStream_t stream);
int smem_optin_of(int device);
// Diagnostic: per-CTA wall-clock phase marks of the last fused launch.
cudaError_t fused_phase_times(unsigned long long* out, int max_ctas, int* n_ctas);

// 2-D tensor map over a row-major array (rows x inner elements, row stride in bytes).
cudaError_t encode_tiled_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
                            uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                            CUtensorMapSwizzle swz);

// prefill path (any M; used for M > 8): tcgen05 GEMMs, Z fp16 [M][k]
cudaError_t prepare_prefill_kernels(int device);
cudaError_t encode_dict_codes_map(const dictproj_group* g, CUtensorMap* map);
// Tile width (multiple of 16, <= 256) for `extent` elements split into tiles,
// `other` tiles along the other side, n_sm SMs (prefill GEMM grids).
int prefill_tile_width(long extent, long other, int n_sm);
// Z = s_D X D^ (fp16 out, s_D applied in fp32 before rounding)
// Grid of the prefill dictionary stage: token-tile width nt and the number of
// CTAs (one cluster) the d_in stages of a tile are split over (1: no split).
struct PrefillDictPlan {
  int nt, splits;
};
PrefillDictPlan prefill_dict_plan(int M, int d_in, int k, int n_sm);
cudaError_t launch_dict_prefill(const dictproj_group* g, const __half* X, int M, __half* Z, cudaStream_t stream);
// Cd[o][a] = C^ densified to fp16 (zeros off the support), [d_out][k]
cudaError_t launch_densify_coeff(const dictproj_layer* l, __half* Cd, cudaStream_t stream);
// Y = s_C Z Cd^T
cudaError_t launch_coeff_prefill(const dictproj_layer* l, const __half* Z, const __half* Cd, int M, __half* Y,
                                 cudaStream_t stream);
cudaError_t take_prefill_error(unsigned int* out);

}  // namespace dictproj
