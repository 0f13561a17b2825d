// Instantiation of the step launcher for storage dtype f32, kind fused.
#include "hc_kernels_impl.cuh"

template hc_status hc::launch_kind<float, hc::KIND_FUSED>(int, const hc::StepParams &,
                                                          const hc::LaunchCtx &, cudaStream_t);
template int hc::step_path<float, hc::KIND_FUSED>(int, const hc::StepParams &, const hc::LaunchCtx &);
