// Instantiates the fp16-input half of the kernel family (104 strip-kernel and
// 36 per-token variants).
#include "pqg_launch.cuh"

namespace pqg {
cudaError_t launch_fp16(const LaunchArgs &a) { return launch_dtype<__half>(a); }
}  // namespace pqg
