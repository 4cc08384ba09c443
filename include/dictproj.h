/*
 * dictproj.h — C ABI of the dictionary-compressed projection library (libdictproj.so).
 *
 * What it computes (DictLLM, arXiv 2611.08082; technical review "DictLLM: Shared
 * Dictionaries for Post-Training Compression", Eq. (1)):
 *
 *     W_l ~= D_g C_l,    Z_l = X_l D_g,    Y_l ~= Z_l C_l
 *
 * Rows of X are tokens. D_g (d_in x k) is a dictionary shared by a group of
 * layers; C_l (k x d_out) is a per-layer coefficient matrix with unstructured
 * sparsity (review, "Prerequisites": each output column may use its own subset
 * of atoms). Both are stored in NVFP4: 4-bit E2M1 values with one 8-bit E4M3
 * scale per block of sixteen values (review, "From retained values to measured
 * decoding": 4.5 bits per value) and one fp32 per-tensor scale.
 *
 * Packed layouts (bit-exact contract; the pages leave them open, so these are
 * plain readings):
 *   D_g:  codes  uint8[k][d_in/2]  element i of atom j at byte j*d_in/2 + i/2, even
 *                                  i in the low nibble (atom-major = K-major);
 *         scales uint8[k][d_in/16] one E4M3 per 16 consecutive d_in entries;
 *         s_D    fp32.
 *   C_l:  column o stores its nnz_o atoms in ascending order, zero-padded to
 *         P_o = 16*ceil(nnz_o/16) entries (code 0, index 0);
 *         col_ptr   uint32[d_out+1]  padded entry offsets;
 *         codes     uint8[total/2]   entry e at byte e/2, even e in the low nibble;
 *         scales    uint8[total/16]  one E4M3 per 16 consecutive stored entries;
 *         idx       uint8[total]     atom mod 256 (the 8-bit index of the review's
 *                                    Eq. (12), a = 8, relative to 256-atom segments);
 *         seg_start uint16[d_out][ceil(k/256)] entry offset (from the column start)
 *                                    of the first entry with atom >= 256*s;
 *         s_C       fp32.
 *   The atom of entry q of a column is 256*s(q) + idx[q], s(q) = max{s : seg_start[s] <= q}.
 *
 * Quantiser used by the packers (round to nearest; the paper's Hessian-aware
 * quantiser needs calibration data and is not part of this library):
 *   s_T = amax/2688 (1 if amax == 0); per block r = amax_b/(6 s_T) rounded to
 *   the nearest E4M3 (ties to even, saturating at 448); each value
 *   x/(E4M3(sc) s_T) rounded to the nearest E2M1 (ties to even mantissa,
 *   saturating at 6, -0 written as 0); a block whose scale is 0 stores zeros.
 *   All arithmetic is IEEE fp32.
 *
 * Conventions for every entry point:
 *   - Returns a dictproj_status (0 = DICTPROJ_OK). Nothing throws across the ABI.
 *     On error a thread-local message is available from dictproj_last_error().
 *   - Arguments are validated before any allocation, copy or kernel launch; an
 *     invalid call has no side effect.
 *   - "host" pointers are ordinary CPU memory; "device" pointers are CUDA device
 *     memory of the device that was current when the handle was created.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - The library owns the memory behind handles; the caller owns everything it
 *     passes in (inputs are only read, outputs only written).
 */
#ifndef DICTPROJ_H
#define DICTPROJ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dictproj_status {
  DICTPROJ_OK = 0,
  DICTPROJ_ERR_NULL = -1,        /* a required pointer is NULL */
  DICTPROJ_ERR_SHAPE = -2,       /* a size is zero, negative or not a multiple of 16 where required */
  DICTPROJ_ERR_ALIGN = -3,       /* X, Y or a caller-owned packed array is not 16-byte aligned */
  DICTPROJ_ERR_MISMATCH = -4,    /* layer and group disagree on k, or live on different devices */
  DICTPROJ_ERR_RANGE = -5,       /* M outside [1, max_tokens], an atom index >= k, unsorted atoms */
  DICTPROJ_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed (or no device) */
  DICTPROJ_ERR_OOM = -7,         /* device or host allocation failed */
  DICTPROJ_ERR_TIMEOUT = -8,     /* a bounded device-side wait gave up (read by dictproj_check) */
  DICTPROJ_ERR_UNSUPPORTED = -9, /* valid but not supported here (e.g. not an sm_100 device) */
  DICTPROJ_ERR_VALUE = -10,      /* a non-finite input value; a corrupt packed file */
  DICTPROJ_ERR_IO = -11          /* a file could not be opened, read or written */
} dictproj_status;

/* Opaque handles. A group owns the packed D_g on the device plus the scratch for
 * Z; a layer owns the packed C_l. Calls that share a group use the group's Z
 * scratch, so they must be ordered on one stream (or otherwise serialised). */
typedef struct dictproj_group dictproj_group;
typedef struct dictproj_layer dictproj_layer;

/* ------------------------------------------------------------------------- */
/* Host-only packing (no GPU needed). Review Algorithm 2, export step: the     */
/* dictionary, per-layer codes, scales and support.                            */
/* ------------------------------------------------------------------------- */

/* Sizes of the packed D_g arrays. d_in % 16 == 0, k >= 1 (the host packers accept
 * any d_in that is a multiple of 16; device groups need d_in % 32 == 0 and
 * k % 16 == 0, see dictproj_group_upload). */
int dictproj_group_packed_sizes(int d_in, int k, size_t* codes_bytes, size_t* scales_bytes);

/* Quantise D (host fp32, d_in x k, row-major) into caller buffers of the sizes
 * above. Errors: NULL, SHAPE, VALUE (non-finite entry). */
int dictproj_pack_group_host(const float* D, int d_in, int k, uint8_t* codes, uint8_t* scales,
                             float* s_D);

/* Total padded entries of C_l given its unpadded CSC column pointers
 * (host int32[d_out+1], col_ptr[0] == 0, non-decreasing, each column <= k entries). */
int dictproj_layer_packed_entries(const int32_t* col_ptr, int k, int d_out, size_t* total_entries);

/* Quantise and lay out C_l (host CSC: col_ptr int32[d_out+1], atom_idx int32[nnz] ascending
 * and unique within each column and < k, vals fp32[nnz]) into caller buffers:
 * pcol_ptr uint32[d_out+1], nnz uint32[d_out], codes uint8[total/2], scales uint8[total/16],
 * idx uint8[total], seg_start uint16[d_out*ceil(k/256)], s_C. k <= 65535.
 * Errors: NULL, SHAPE, RANGE (bad index or order), VALUE (non-finite value). */
int dictproj_pack_layer_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals,
                             int k, int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes,
                             uint8_t* scales, uint8_t* idx, uint16_t* seg_start, float* s_C);

/* The same C_l with a bitmap support index instead of idx + seg_start: the
 * review's Eq. (12) case a = 0, h = 1 (one bit per logical position; it saves
 * bytes over the 8-bit index for every density above 1/8 and over dense NVFP4
 * above 22.2% sparsity). Codes, scales, padding, pcol_ptr, nnz and s_C are
 * exactly those of dictproj_pack_layer_host; bitmap is uint32[d_out][ceil(k/32)]
 * with bit j % 32 of word j / 32 of row o set iff atom j is retained in column o
 * (the set bits, ascending, are the column's stored entries in storage order;
 * padding entries have no bit). Errors as dictproj_pack_layer_host. */
int dictproj_pack_layer_bitmap_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals,
                                    int k, int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes,
                                    uint8_t* scales, uint32_t* bitmap, float* s_C);

/* C_l with block-structured support (review, "Let the accelerator constrain
 * the support"; block-structured sparsity is the paper's named future work):
 * every column's retained atoms are whole aligned blocks of 16 consecutive
 * atoms (col_ptr / atom_idx as for dictproj_pack_layer_host, each column a union
 * of such blocks). A kept block is one NVFP4 block, so codes and scales are
 * exactly those of dictproj_pack_layer_host on the same support (no padding is
 * needed); the index is one uint16 block number (atom / 16) per kept block:
 *   blk_ptr uint32[d_out+1]  kept blocks before each column;
 *   blk_idx uint16[nblk]     ascending within a column;
 *   codes uint8[nblk*8], scales uint8[nblk], s_C fp32.
 * Errors as dictproj_pack_layer_host, plus RANGE (a column that is not a union of
 * aligned 16-atom blocks). */
int dictproj_pack_layer_blocks_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals,
                                    int k, int d_out, uint32_t* blk_ptr, uint16_t* blk_idx, uint8_t* codes,
                                    uint8_t* scales, float* s_C);

/* Support index formats of a device layer (DICTPROJ_IFMT_*): the u8
 * segment-relative index with seg_start (the default layout above), the bitmap
 * of dictproj_pack_layer_bitmap_host, or the 16-atom blocks of
 * dictproj_pack_layer_blocks_host. Bitmap and block layers hold NVFP4 values and
 * are served by the two-kernel decode path (their own coefficient kernels; Z of
 * k * mp floats in shared memory, mp = the power of two >= M) and by the
 * prefill path (their own densify kernels, the same GEMM); the fused decode
 * kernel, dictproj_layer_export and dictproj_layer_save take u8 layers only
 * (UNSUPPORTED otherwise). */
enum { DICTPROJ_IFMT_U8 = 0, DICTPROJ_IFMT_BITMAP = 1, DICTPROJ_IFMT_BLOCKS = 2 };

/* Upload a bitmap C_l (the arrays of dictproj_pack_layer_bitmap_host) to the
 * current device. Validation: k % 16 == 0, 0 < k <= 65535, d_out > 0; col_ptr[0]
 * == 0, columns padded to multiples of 16 with less than 16 padding entries
 * beyond their set bits; no bit at atoms >= k; s_C finite and > 0 (else SHAPE /
 * RANGE / VALUE). Errors also NULL, OOM, CUDA. */
int dictproj_layer_upload_bitmap(const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                                 const uint32_t* bitmap, float s_C, int k, int d_out, dictproj_layer** out);
/* dictproj_pack_layer_bitmap_host + dictproj_layer_upload_bitmap. */
int dictproj_pack_layer_bitmap(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                               int d_out, dictproj_layer** out);

/* Upload a block-structured C_l (the arrays of dictproj_pack_layer_blocks_host,
 * nblk = blk_ptr[d_out]; codes nblk*8 bytes, scales nblk bytes). Validation:
 * blk_ptr[0] == 0 and non-decreasing with at most k/16 blocks per column; block
 * numbers ascending per column and below k/16 (RANGE); shape and s_C as
 * dictproj_layer_upload_bitmap. */
int dictproj_layer_upload_blocks(const uint32_t* blk_ptr, const uint16_t* blk_idx, const uint8_t* codes,
                                 const uint8_t* scales, float s_C, int k, int d_out, dictproj_layer** out);
/* dictproj_pack_layer_blocks_host + dictproj_layer_upload_blocks (VALUE / RANGE
 * when a column's support is not a union of aligned 16-atom blocks). */
int dictproj_pack_layer_blocks(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                               int d_out, dictproj_layer** out);

/* The support index format of a layer (DICTPROJ_IFMT_*). Errors: NULL. */
int dictproj_layer_index_format(const dictproj_layer* l, int* ifmt);

/* Copy a bitmap / block layer's arrays back to host buffers of their packed
 * sizes (bitmap: d_out * ceil(k/32) words). Errors: NULL, UNSUPPORTED (the other
 * index format), CUDA. */
int dictproj_layer_export_bitmap(const dictproj_layer* l, uint32_t* pcol_ptr, uint8_t* codes, uint8_t* scales,
                                 uint32_t* bitmap, float* s_C);
int dictproj_layer_export_blocks(const dictproj_layer* l, uint32_t* blk_ptr, uint16_t* blk_idx, uint8_t* codes,
                                 uint8_t* scales, float* s_C);

/* Coefficient value formats: NVFP4 (the default layout above) and the three
 * other coefficient formats of the paper's Table 4 (with an NVFP4 dictionary). */
enum { DICTPROJ_CFMT_NVFP4 = 0, DICTPROJ_CFMT_FP16 = 1, DICTPROJ_CFMT_FP8 = 2, DICTPROJ_CFMT_INT8 = 3 };

/* Bytes of one stored coefficient value in format fmt (NVFP4: 0, it packs two
 * per byte plus a scale per 16; see dictproj_pack_layer_host). */
int dictproj_cfmt_value_bytes(int fmt);

/* C_l with its values in FP16, FP8 or INT8 (Table 4) and the index of the NVFP4
 * layout: pcol_ptr, nnz, idx and seg_start exactly as dictproj_pack_layer_host
 * writes them; values holds one code per stored entry (padding entries 0):
 *   DICTPROJ_CFMT_FP16  uint16 binary16 bits of x (round to nearest even), s_C = 1;
 *   DICTPROJ_CFMT_FP8   uint8 E4M3FN: sign | the magnitude code nearest to |x| / s_C
 *                       (ties to even, saturating at 448), s_C = amax / 448;
 *   DICTPROJ_CFMT_INT8  int8 nearest integer to x / s_C (ties to even), clamped to
 *                       [-127, 127], s_C = amax / 127 (s_C = 1 if amax = 0).
 * Value = s_C * decoded code. values: total_entries codes of
 * dictproj_cfmt_value_bytes(fmt) bytes. Errors: NULL, SHAPE, RANGE (format, index,
 * order), VALUE (non-finite value; an FP16 value beyond 65504). */
int dictproj_pack_layer_fmt_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                                 int d_out, int fmt, uint32_t* pcol_ptr, uint32_t* nnz, void* values,
                                 uint8_t* idx, uint16_t* seg_start, float* s_C);

/* ------------------------------------------------------------------------- */
/* Device objects                                                             */
/* ------------------------------------------------------------------------- */

/* Upload an already packed D_g (host arrays as produced above) to the current
 * device and allocate the Z scratch for up to max_tokens tokens per call.
 * Shapes: d_in % 32 == 0, k % 16 == 0, 1 <= k <= 65535.
 * Errors: NULL, SHAPE, RANGE (max_tokens < 1), CUDA, OOM. */
int dictproj_group_upload(const uint8_t* codes, const uint8_t* scales, float s_D, int d_in, int k,
                          int max_tokens, dictproj_group** out);

/* dictproj_pack_group_host + dictproj_group_upload. */
int dictproj_pack_group(const float* D, int d_in, int k, int max_tokens, dictproj_group** out);

/* Reserve the group's prefill coefficient scratch for layers with up to max_d_out
 * output columns: fp16 [max_d_out][k], the densified C_l that the prefill
 * coefficient GEMM reads (2 * k * max_d_out bytes). Forwards with M > 8 (or
 * DICTPROJ_PATH_PREFILL) need it and fail with RANGE before any launch without
 * it, so that they never allocate. Growing an existing reservation synchronises
 * the device first. dictproj_pack reserves for its layers when max_tokens > 8.
 * Errors: NULL, RANGE (max_d_out < 1), MISMATCH (device), OOM, CUDA. */
int dictproj_group_reserve_prefill(dictproj_group* g, int max_d_out);

/* Upload an already packed C_l. Errors: NULL, SHAPE, CUDA, OOM. */
int dictproj_layer_upload(const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                          const uint8_t* idx, const uint16_t* seg_start, float s_C, int k,
                          int d_out, dictproj_layer** out);

/* dictproj_pack_layer_host + dictproj_layer_upload. */
int dictproj_pack_layer(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                        int d_out, dictproj_layer** out);

/* A C_l with FP16 / FP8 / INT8 values (dictproj_pack_layer_fmt_host's arrays,
 * `values` of dictproj_cfmt_value_bytes(fmt) bytes per stored entry) on the
 * current device. Such a layer is decoded by the fused decode kernel
 * (M <= 8, k <= 8192) and by the prefill path; other calls with it
 * return UNSUPPORTED before any launch. dictproj_layer_save refuses it (the
 * packed file holds NVFP4 layers). Errors as dictproj_layer_upload, plus RANGE
 * (fmt not FP16 / FP8 / INT8). */
int dictproj_layer_upload_fmt(const uint32_t* pcol_ptr, const void* values, const uint8_t* idx,
                              const uint16_t* seg_start, float s_C, int k, int d_out, int fmt,
                              dictproj_layer** out);

/* dictproj_pack_layer_fmt_host + dictproj_layer_upload_fmt (fmt NVFP4: dictproj_pack_layer). */
int dictproj_pack_layer_fmt(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                            int d_out, int fmt, dictproj_layer** out);

/* The coefficient value format of a layer (DICTPROJ_CFMT_*). Errors: NULL. */
int dictproj_layer_format(const dictproj_layer* l, int* fmt);

/* Copy an FP16 / FP8 / INT8 layer's packed arrays back to host buffers of the
 * packed sizes. Errors: NULL, UNSUPPORTED (an NVFP4 layer), CUDA. */
int dictproj_layer_export_fmt(const dictproj_layer* l, uint32_t* pcol_ptr, void* values, uint8_t* idx,
                              uint16_t* seg_start, float* s_C);

/* Convenience: pack one group and its n_layers layers (all with the same k).
 * On error nothing is left allocated. */
int dictproj_pack(const float* D, int d_in, int k, int max_tokens, int n_layers,
                  const int32_t* const* col_ptr, const int32_t* const* atom_idx,
                  const float* const* vals, const int* d_out, dictproj_group** group_out,
                  dictproj_layer** layers_out);

/* Copy the packed bytes back to host buffers of the packed sizes (for
 * bit-exact checks). Errors: NULL, UNSUPPORTED (a layer whose values are not
 * NVFP4: dictproj_layer_export_fmt), CUDA. */
int dictproj_group_export(const dictproj_group* g, uint8_t* codes, uint8_t* scales, float* s_D);
int dictproj_layer_export(const dictproj_layer* l, uint32_t* pcol_ptr, uint8_t* codes,
                          uint8_t* scales, uint8_t* idx, uint16_t* seg_start, float* s_C);

/* Shape queries. Any output pointer may be NULL. */
int dictproj_group_info(const dictproj_group* g, int* d_in, int* k, int* max_tokens);
int dictproj_layer_info(const dictproj_layer* l, int* k, int* d_out, size_t* total_entries,
                        size_t* nnz_total);

void dictproj_free_group(dictproj_group* g); /* NULL is a no-op */
void dictproj_free_layer(dictproj_layer* l); /* NULL is a no-op */

/* ------------------------------------------------------------------------- */
/* Forward                                                                    */
/* ------------------------------------------------------------------------- */

/* Y = X * (D_g) * (C_l) (Eq. (1)): X device fp16 [M][d_in] row-major, Y device
 * fp16 [M][d_out] row-major, both 16-byte aligned; 1 <= M <= group max_tokens.
 * Accumulation is fp32; Z is fp32 for M <= 8 (decode path: the dictionary GEMV on
 * mma.sync tensor-core instructions, then the sparse gather on CUDA cores, which
 * stages (k + 256) * mp floats of Z in shared memory, mp = 1, 2, 4 or 8 the
 * smallest power of two >= M; k above 57856 / 28800 / 14272 / 7008 for
 * mp = 1 / 2 / 4 / 8 does not fit the 227 KiB per-block limit and returns
 * UNSUPPORTED before any launch) and fp16 with s_D applied before rounding for larger M (prefill
 * path: tcgen05 GEMM on the dequantised dictionary, then the densified C_l as a
 * second tcgen05 GEMM; needs dictproj_group_reserve_prefill for d_out).
 * Asynchronous on `stream`: no allocation, no host synchronisation. Kernels are
 * launched with programmatic dependent launch; each kernel waits for the
 * preceding work on the stream before it reads X or writes Z / Y (packed
 * weights, which nothing writes after upload, may be prefetched earlier). A group
 * serves one stream at a time: its Z scratch is shared by its calls.
 * Errors (checked before any launch): NULL, RANGE (M), MISMATCH (k or device),
 * ALIGN, UNSUPPORTED (k too large for the decode path's shared memory); CUDA if
 * a launch fails. */
int dictproj_forward(const void* X, int M, const dictproj_layer* layer,
                     const dictproj_group* group, void* Y, void* stream);

/* Up to DICTPROJ_MAX_BATCH independent projections in one call: projection i
 * computes Y[i] = X[i] D_g[i] C_l[i] with the kernels and arithmetic of
 * dictproj_forward. The dictionary stage's d_in slicing is planned over the whole
 * batch (dictproj_decode_batch_plan), so Y[i] equals dictproj_forward's bit for
 * bit where that plan gives projection i the slices it gets alone, and otherwise
 * agrees within the decode tolerance (its fp32 partial sums split differently). The projections must be
 * independent: no Y[i] may be read as an X[j] of the same call; X entries may
 * alias (e.g. the q, k and v projections of one layer read the same activation);
 * the groups must be distinct (each call uses its group's Z scratch). For
 * M <= 8 all projections share one launch per stage, which shortens the chain of
 * dependent launches a decode step pays; larger M runs them one after another.
 * Errors as dictproj_forward, plus RANGE (n outside [1, DICTPROJ_MAX_BATCH]) and
 * MISMATCH (a group repeated or M above some group's max_tokens). */
#define DICTPROJ_MAX_BATCH 4
int dictproj_forward_batch(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                           const dictproj_group* const* groups, void* const* Y, void* stream);

/* dictproj_forward_batch with a stage mask, to time each kernel of the two-kernel
 * decode path in the launch configuration a full call uses (the same batch plan,
 * grids and Z scratch): bit 0 launches the dictionary kernel (Z = X D_g into each
 * group's Z scratch), bit 1 the coefficient kernel (Y = Z C_l from that scratch,
 * as the last dictionary launch on these groups left it); 3 is the full call.
 * A mask of 1 or 2 needs M <= 8 and a call the two-kernel path serves.
 * Errors as dictproj_forward_batch, plus RANGE (mask not 1, 2 or 3) and
 * UNSUPPORTED (a mask of 1 or 2 with M > 8 or on the fused kernel). */
int dictproj_forward_batch_stages(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                                  const dictproj_group* const* groups, void* const* Y, void* stream, int stages);

/* The grid a batched two-kernel decode call (1 <= M <= 8) of n <= DICTPROJ_MAX_BATCH
 * projections would launch, host only: projection i has d_in[i] rows, k[i] atoms,
 * d_out[i] columns and entries[i] stored (padded) coefficient entries; n_sm is
 * the device's SM count. Out (caller-owned arrays of n ints): dict_ctas[i] and
 * dict_slices[i], the dictionary kernel's CTAs and d_in slices for projection i
 * (every CTA streams the same number of dictionary rows, so CTAs follow
 * d_in x k), and coeff_ctas[i], the coefficient kernel's CTAs for projection i
 * (n_sm in all before rounding columns up, at least one each, handed out one at a
 * time to the projection whose CTAs would finish last by a cost of whole columns
 * per warp, each column a fixed part worth two 256-entry windows plus its
 * windows; equal projections get equal shares).
 * Errors: NULL, RANGE (n, M, n_sm, entries < 0), SHAPE. */
int dictproj_decode_batch_plan(int n, const int* d_in, const int* k, const int* d_out, const long long* entries,
                               int M, int n_sm, int* dict_ctas, int* dict_slices, int* coeff_ctas);

/* Number of kernels that dictproj_forward_batch with these arguments (n = 1:
 * dictproj_forward) launches: 1 for a decode call served by the fused kernel,
 * 2 (or 1 + n) on the two-kernel decode path, 3 per projection at prefill.
 * Host only; nothing is launched. Errors: NULL, RANGE. */
int dictproj_launch_count(int n, const void* const* X, int M, const dictproj_layer* const* layers,
                          const dictproj_group* const* groups, int* count);

/* Which kernels serve decode calls (M <= 8), process-wide (default AUTO):
 *   DICTPROJ_DECODE_AUTO   the two-kernel path, which is the faster one on B200 for every
 *                          LLaMA-7B shape measured, and the fused kernel for calls the
 *                          two-kernel path cannot serve (FP16 / FP8 / INT8 coefficient
 *                          values, or a Z table beyond its shared memory);
 *   DICTPROJ_DECODE_FUSED  the single fused kernel only; a call it cannot serve (k > 8192,
 *                          or its shared memory plan does not fit) fails with UNSUPPORTED;
 *   DICTPROJ_DECODE_SPLIT  the two-kernel path only (dictionary stage, then coefficient
 *                          stage); NVFP4 coefficients only, else UNSUPPORTED.
 * Both compute the same function within the same tolerance (their fp32 summation
 * orders differ). Set it between calls, not while another thread enqueues work.
 * Errors: RANGE (unknown value). */
enum { DICTPROJ_DECODE_AUTO = 0, DICTPROJ_DECODE_FUSED = 1, DICTPROJ_DECODE_SPLIT = 2 };
int dictproj_set_decode_kernels(int which);
int dictproj_get_decode_kernels(void);

/* Forward with an explicit path: DICTPROJ_PATH_AUTO, DICTPROJ_PATH_DECODE (M <= 8)
 * or DICTPROJ_PATH_PREFILL (any M). Errors as dictproj_forward, plus
 * UNSUPPORTED for DECODE with M > 8. */
enum { DICTPROJ_PATH_AUTO = 0, DICTPROJ_PATH_DECODE = 1, DICTPROJ_PATH_PREFILL = 2 };
int dictproj_forward_path(const void* X, int M, const dictproj_layer* layer,
                          const dictproj_group* group, void* Y, void* stream, int path);

/* The two stages of Eq. (1) as separate calls (decode path, 1 <= M <= 8).
 * Z is caller-owned device fp32 [k][mp], 16-byte aligned, mp = 1, 2, 4 or 8 = the
 * smallest power of two >= M; column m of Z holds token m (columns >= M are zero).
 *   dictionary stage:   Z = X D_g        (X device fp16 [M][d_in])
 *   coefficient stage:  Y = Z C_l        (Y device fp16 [M][d_out])
 * Same validation, ordering and asynchrony as dictproj_forward; UNSUPPORTED for M > 8. */
int dictproj_dictionary_stage(const void* X, int M, const dictproj_group* group, float* Z, void* stream);
int dictproj_coefficient_stage(const float* Z, int M, const dictproj_layer* layer, void* Y, void* stream);

/* The prefill dictionary stage alone (any M >= 1): Z = s_D * X * D_g on tcgen05
 * tensor cores (fp16 operands, fp32 accumulation, s_D applied in fp32, then
 * rounded to fp16). X device fp16 [M][d_in], Z caller-owned device fp16 [M][k],
 * both 16-byte aligned. Same ordering and asynchrony as dictproj_forward.
 * Errors: NULL, RANGE (M < 1), ALIGN, MISMATCH (device), CUDA. */
int dictproj_dictionary_stage_prefill(const void* X, int M, const dictproj_group* group, void* Z, void* stream);

/* ------------------------------------------------------------------------- */
/* Forward without allocation                                                 */
/* ------------------------------------------------------------------------- */

/* Caller-owned device copies of packed factors (the arrays produced by
 * dictproj_pack_group_host / dictproj_pack_layer_host, copied to the device by
 * the caller). All pointers are device pointers, each 16-byte aligned (the
 * kernels use 16-byte vector loads and 16-byte L2 prefetches); the library only
 * reads them. */
typedef struct dictproj_device_group {
  const uint8_t* codes;   /* [k][d_in/2] */
  const uint8_t* scales;  /* [k][d_in/16] */
  float s;                /* s_D */
  int d_in, k;
} dictproj_device_group;

typedef struct dictproj_device_layer {
  const uint32_t* col_ptr;    /* [d_out+1] */
  const uint8_t* codes;       /* [total/2] */
  const uint8_t* scales;      /* [total/16] */
  const uint8_t* idx;         /* [total] */
  const uint16_t* seg_start;  /* [d_out][ceil(k/256)] */
  float s;                    /* s_C */
  int k, d_out;
} dictproj_device_layer;

/* The decode-path forward (1 <= M <= 8) for callers that cannot allocate device
 * memory at call time: runtimes that reserve all device memory up front in their
 * own arena, and code enqueuing work while a stream is captured into a CUDA graph.
 * It computes the same Y = X D_g C_l as dictproj_forward; the paper has no
 * counterpart for this entry point (it is an integration convenience).
 * Nothing is allocated: the Z scratch between the two stages is a file-scope
 * device array of 49152 floats (192 KiB) that every GPU loading the library holds
 * until exit; (k + 256) * mp must not exceed 49152, where mp = 1, 2, 4 or 8 is the
 * smallest power of two >= M, else DICTPROJ_ERR_RANGE and nothing is launched.
 * The first call with a given device current resolves the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture. All
 * calls share the array: calls that overlap on the GPU race and must be
 * serialised by the caller. X fp16 [M][d_in], Y fp16 [M][d_out], both device,
 * 16-byte aligned. Errors: NULL, SHAPE, MISMATCH, RANGE, ALIGN (X, Y or any packed
 * array not 16-byte aligned), VALUE, CUDA. */
int dictproj_forward_noalloc(const dictproj_device_group* group, const dictproj_device_layer* layer,
                             const void* X, int M, void* Y, void* stream);

/* ------------------------------------------------------------------------- */
/* Budget helpers and packed-file export (host only, no device needed)        */
/* ------------------------------------------------------------------------- */

/* Rank of a group's dictionary for a factorisation budget, Eq. (3) of the
 * DictLLM technical review ("The budget: trading shared rank against
 * sparsity"): k = floor((1 - rho_fac) n d_in d_out / (d_in + n d_out)) for n
 * layers of shape d_in x d_out, rounded down to a multiple of `align` (1 for
 * the plain equation; 16 for the kernels here, which need k % 16 == 0).
 * Errors: NULL, SHAPE (n, d_in, d_out, align < 1), RANGE (rho_fac outside
 * [0, 1), or no rank left). */
int dictproj_rank_for_budget(double rho_fac, int n, int d_in, int d_out, int align, int* k_out);

/* Value counts of Eq. (2) of the review: N0 = n d_in d_out, Np = d_in k +
 * n (1 - p) k d_out, rho = 1 - Np / N0, G = N0 / Np (p = fraction of the
 * coefficients pruned). Any output may be NULL. Errors: SHAPE, RANGE (p). */
int dictproj_budget(int n, int d_in, int d_out, int k, double p, double* N0, double* Np, double* rho, double* G);

/* Packed-file export and import of one group (D_g) or one layer (C_l): the
 * export step of the review's Algorithm 2 ("dictionary, per-layer codes, scales
 * and support"). A file holds exactly the packed arrays of
 * dictproj_pack_group_host / dictproj_pack_layer_host behind a 64-byte header
 * (magic, shapes, the fp32 tensor scale, payload size, FNV-1a 64 checksum),
 * little-endian. *_info reads the shapes so that the caller can size buffers;
 * *_read checks magic, shapes against the caller's, sizes and the checksum.
 * Errors: NULL, SHAPE, RANGE (bad layout on write), VALUE (non-finite scale;
 * corrupt, truncated or foreign file), MISMATCH (buffer shapes), IO. */
int dictproj_group_file_write(const char* path, const uint8_t* codes, const uint8_t* scales, float s_D, int d_in,
                              int k);
int dictproj_group_file_info(const char* path, int* d_in, int* k);
int dictproj_group_file_read(const char* path, uint8_t* codes, uint8_t* scales, float* s_D, int d_in, int k);
int dictproj_layer_file_write(const char* path, const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                              const uint8_t* idx, const uint16_t* seg_start, float s_C, int k, int d_out);
int dictproj_layer_file_info(const char* path, int* k, int* d_out, size_t* total_entries);
int dictproj_layer_file_read(const char* path, uint32_t* pcol_ptr, uint8_t* codes, uint8_t* scales, uint8_t* idx,
                             uint16_t* seg_start, float* s_C, int k, int d_out, size_t total_entries);

/* Device handles to and from packed files: *_save exports the handle's packed
 * bytes (dictproj_*_export) and writes them; *_load reads a file and uploads it
 * (dictproj_group_upload / dictproj_layer_upload, which validate the layout).
 * Errors: those of the calls they compose. */
int dictproj_group_save(const dictproj_group* g, const char* path);
int dictproj_group_load(const char* path, int max_tokens, dictproj_group** out);
int dictproj_layer_save(const dictproj_layer* l, const char* path);
int dictproj_layer_load(const char* path, dictproj_layer** out);

/* Read (and clear) the device error word that bounded device waits set, after
 * synchronising `stream`. Returns OK or TIMEOUT (or CUDA). */
int dictproj_check(void* stream);

/* Diagnostic (no counterpart in the paper): wall-clock marks (ns, the GPU's
 * global timer) at the phase boundaries of the most recent fused decode launch,
 * per CTA: out[cta * 16 + slot] for cta < min(max_ctas, 1024); *n_ctas = rows
 * written. Slots 0-7 (compute warps): start, dependency resolved, X staged,
 * dictionary stage done, partial Z published, exchange passed, Z tables loaded,
 * end; 8-11 (producer): first slots issued, dependents released, dependency
 * resolved, last copy issued; 12-15 unused. Synchronise the stream first.
 * Errors: NULL, RANGE, UNSUPPORTED, CUDA. */
int dictproj_diag_phase_times(unsigned long long* out, int max_ctas, int* n_ctas);

/* Diagnostic (no counterpart in the paper): while armed, every launch of the
 * decode gather kernel (the coefficient stage of the two-kernel path) writes, for
 * each of its CTAs c < max_ctas, the GPU's global timer (ns) when the CTA's
 * column work starts (its Z table staged) to buf[2c] and at its end to
 * buf[2c + 1]. buf is caller-owned device memory of 2 * max_ctas u64, 8-byte
 * aligned; buf = NULL disarms. The CTAs of a batched launch are the projections'
 * CTAs in order (dictproj_decode_batch_plan gives how many each has). Set it
 * between calls, not while kernels run.
 * Errors: RANGE (max_ctas < 1 with a buffer), ALIGN, UNSUPPORTED, CUDA. */
int dictproj_diag_gather_times(unsigned long long* buf, int max_ctas);

/* Self-test of the bounded-wait error path (diagnostic; no counterpart in the
 * paper). Launches, on `stream`, one warp per kernel file (decode, prefill, fused
 * decode: each has its own device error word) that waits on an mbarrier which
 * can never complete, with a limit of `cycles` SM clocks (1 <= cycles <= 2^31).
 * Each wait gives up at the limit, sets its file's error word and the kernel
 * returns; no copy or tensor-core operation is in flight. A following dictproj_check(stream)
 * then returns DICTPROJ_ERR_TIMEOUT and clears the word; the device stays usable.
 * Errors: RANGE (cycles), UNSUPPORTED (not sm_100), CUDA. */
int dictproj_selftest_wait_timeout(long long cycles, void* stream);

/* Last error message of the calling thread ("" if none). */
const char* dictproj_last_error(void);
/* Static name of a status code. */
const char* dictproj_status_string(int status);
/* Library ABI version (major*10000 + minor*100 + patch). */
int dictproj_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DICTPROJ_H */
