// Instantiation of the step launcher for storage dtype bf16, kind read.
#include "hc_kernels_impl.cuh"

template hc_status hc::launch_kind<__nv_bfloat16, hc::KIND_READ>(int, const hc::StepParams &,
                                                          const hc::LaunchCtx &, cudaStream_t);
template int hc::step_path<__nv_bfloat16, hc::KIND_READ>(int, const hc::StepParams &, const hc::LaunchCtx &);
