// Instantiates the bf16-input half of the kernel family (104 strip-kernel and
// 36 per-token variants).
#include "pqg_launch.cuh"

namespace pqg {
cudaError_t launch_bf16(const LaunchArgs &a) { return launch_dtype<__nv_bfloat16>(a); }
}  // namespace pqg
