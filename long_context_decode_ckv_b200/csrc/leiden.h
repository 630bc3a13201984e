// leiden.h -- host graph partition and device modularity of libckv.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ckv {

// Leiden partition of the directed top-kappa CSR read as an undirected
// weighted graph (leiden.cpp); labels get 0..C-1 by first appearance;
// returns C.
int leiden_partition(int n, const int64_t* row_ptr, const int32_t* col, const float* w, double gamma,
                     int max_levels, int32_t* labels);

// modularity with resolution gamma of a labelling of that graph, on the
// device (k_modularity.cu): scratch = modularity_scratch_doubles(nc) doubles
size_t modularity_scratch_doubles(int n_communities);
cudaError_t launch_modularity(int n, const int64_t* row_ptr, const int32_t* col, const float* w,
                              const int32_t* labels, int n_communities, double gamma, double* scratch,
                              double* q_out, cudaStream_t st);

}  // namespace ckv
