// Instantiation of the step launcher for storage dtype bf16, kind fused.
#include "hc_kernels_impl.cuh"

template hc_status hc::launch_kind<__nv_bfloat16, hc::KIND_FUSED>(int, const hc::StepParams &,
                                                          const hc::LaunchCtx &, cudaStream_t);
template int hc::step_path<__nv_bfloat16, hc::KIND_FUSED>(int, const hc::StepParams &, const hc::LaunchCtx &);
