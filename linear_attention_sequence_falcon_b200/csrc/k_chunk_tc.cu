// k_chunk_tc.cu -- bf16 chunk-parallel forward on the tcgen05 tensor cores.
#include "common.cuh"
#include "kernels.h"

namespace falcon {

int launch_tc_chunk(const FwdParams &, cudaStream_t) { return 1; }

}  // namespace falcon
