// Instantiation of the pipelined fused all-reduce write for storage dtype f32.
#include "hc_kernels_impl.cuh"

template hc_status hc::launch_reduce_pipe<float>(const hc::ReduceWriteArgs &, const bool *,
                                                 const hc::LaunchCtx &, cudaStream_t, bool *);
