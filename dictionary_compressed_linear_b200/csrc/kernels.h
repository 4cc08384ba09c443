// Kernel launchers (host side), one per stage and path.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <vector>

#include "dictproj_internal.h"

namespace dictproj {

// decode path (M <= 8): Z fp32 [k][mp], mp = next power of two >= M (at most 8)
int decode_mp(int M);
size_t coeff_decode_smem(int k, int mp);
cudaError_t prepare_decode_kernels(int device);
cudaError_t launch_dict_decode(const dictproj_group* g, const __half* X, int M, int mp, float* Z,
                               cudaStream_t stream);
cudaError_t launch_coeff_decode(const dictproj_layer* l, const float* Z, int M, int mp, __half* Y,
                                cudaStream_t stream);

// Work plan of the chunked coefficient kernel for a grid of G CTAs (host side).
bool plan_coeff_chunks(const uint32_t* pcol_ptr, int d_out, int nseg, int G, std::vector<uint32_t>& chunks,
                       std::vector<int>& cta_ptr);
// Read and clear the device error word of the decode kernels.
cudaError_t take_decode_error(unsigned int* out);

}  // namespace dictproj
