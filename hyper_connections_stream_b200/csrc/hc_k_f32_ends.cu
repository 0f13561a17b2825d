// Instantiation of the stack-end launchers (expand, expand + read, collapse)
// for storage dtype f32.
#include "hc_kernels_impl.cuh"

template hc_status hc::launch_kind<float, hc::KIND_EXPAND>(int, const hc::StepParams &,
                                                       const hc::LaunchCtx &, cudaStream_t);
template hc_status hc::launch_kind<float, hc::KIND_EXPAND_READ>(int, const hc::StepParams &,
                                                            const hc::LaunchCtx &, cudaStream_t);
template hc_status hc::launch_kind<float, hc::KIND_COLLAPSE>(int, const hc::StepParams &,
                                                         const hc::LaunchCtx &, cudaStream_t);
