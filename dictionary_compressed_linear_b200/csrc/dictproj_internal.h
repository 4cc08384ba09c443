// Internal declarations shared by the host packer, the ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "dictproj.h"

namespace dictproj {

// Record a formatted error message for dictproj_last_error() and return `status`.
int fail(int status, const char* fmt, ...)
#if defined(__GNUC__)
    __attribute__((format(printf, 2, 3)))
#endif
    ;
void clear_error();
// Record a CUDA failure (DICTPROJ_ERR_CUDA) with the call that failed.
int cuda_fail(cudaError_t e, const char* what);
// Check the current device (sm_100) and set kernel attributes once per device;
// allocates nothing.
int ensure_device(int* dev_out);

int pack_group_host(const float* D, int d_in, int k, uint8_t* codes, uint8_t* scales, float* s_D);
int layer_packed_entries(const int32_t* col_ptr, int k, int d_out, size_t* total);
int pack_layer_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                    int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes, uint8_t* scales,
                    uint8_t* idx, uint16_t* seg_start, float* s_C);
int pack_layer_fmt_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                        int fmt, uint32_t* pcol_ptr, uint32_t* nnz, void* values, uint8_t* idx,
                        uint16_t* seg_start, float* s_C);
int pack_layer_blocks_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                           uint32_t* blk_ptr, uint16_t* blk_idx, uint8_t* codes, uint8_t* scales, float* s_C);
int pack_layer_bitmap_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                           uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes, uint8_t* scales, uint32_t* bitmap,
                           float* s_C);

// Largest M served by the decode (GEMV) path.
constexpr int kDecodeMaxTokens = 8;

// Default limit of a bounded device wait: 2^31 SM clocks (about one second).
constexpr long long kWaitLimitCycles = 1ll << 31;

}  // namespace dictproj

// Device-side state behind the opaque handles.
struct dictproj_group {
  int device;
  int d_in, k, max_tokens;
  float s;                 // s_D
  uint8_t* codes;          // [k][d_in/2]
  uint8_t* scales;         // [k][d_in/16]
  size_t codes_bytes, scales_bytes;
  int n_sm;                // SMs of the device (sizes the decode grid)
  // scratch
  float* z32;              // decode Z partial sums, fp32 [zslices][k][8]
  int zslices;             // d_in slices of the decode dictionary stage
  uint16_t* z16;           // prefill Z, fp16 [max_tokens][k]
  uint16_t* cdense;        // prefill coefficient operand, fp16 [d_out][k] for d_out <= cdense_cols
  int cdense_cols;         // reserved output columns (dictproj_group_reserve_prefill)
  CUtensorMap codes_map;   // TMA map of codes: [k] rows x [d_in/2] bytes, box 32 x 256
  // fused decode kernel
  bool fused_ok;           // the fused kernel serves this group
  uint8_t* fcodes;         // tile-major copy of the codes: [16-atom tile][512-element piece][16 rows][256 B]
  uint8_t* fscales;        // tile-major copy of the scales: [tile][piece][16 rows][32 B]
  unsigned long long* zx;  // partial-Z exchange buffer [zslots][k][mp] of (tag << 32 | fp32 bits)
  int zslots;              // CTAs one 16-atom tile is split over, at most
  int ppr;                 // 512-element pieces per atom row
  int tp_bound;            // tiles one CTA's pieces span, at most
  unsigned long long* fsync;  // [0] launch ticket of the exchange buffer (one per CTA per launch)
};

struct dictproj_layer {
  int device;
  int k, d_out, nseg;
  float s;                 // s_C
  size_t total;            // padded entries
  size_t nnz_total;        // true entries
  uint32_t* col_ptr;       // [d_out+1]
  uint8_t* codes;          // [total/2]
  uint8_t* scales;         // [total/16]
  uint8_t* idx;            // [total]
  uint16_t* seg_start;     // [d_out][nseg]
  int n_sm;                // SMs of the device
  bool gather_ok;          // the gather kernel serves this layer (else the direct kernel)
  int cfmt;                // coefficient value format: NVFP4 (codes + scales) or FP16 / FP8 / INT8 (codes = values)
  int ifmt;                // support index format (DICTPROJ_IFMT_*): u8 idx + seg_start, bitmap, or 16-atom blocks
  uint32_t* bitmap;        // bitmap layers: [d_out][words] retained-atom masks
  int words;               // 32-bit words per bitmap row, ceil(k/32)
  uint32_t* blk_ptr;       // block layers: [d_out+1] kept blocks before each column
  uint16_t* blk_idx;       // block layers: [nblk] block number (atom / 16), ascending per column
  size_t nblk;             // block layers: kept blocks
  // fused decode kernel: column chunks of each of the n_sm positions
  bool fused_ok;
  uint32_t* cplan_off;     // [n_sm + 1]
  uint4* cplan;            // {o_a, o_b, E_a, E_b}
  int cplan_max;           // chunks of the busiest position
};
