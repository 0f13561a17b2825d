// Instantiation of the pipelined fused all-reduce write for storage dtype bf16.
#include "hc_kernels_impl.cuh"

template hc_status hc::launch_reduce_pipe<__nv_bfloat16>(const hc::ReduceWriteArgs &, const bool *,
                                                 const hc::LaunchCtx &, cudaStream_t, bool *);
