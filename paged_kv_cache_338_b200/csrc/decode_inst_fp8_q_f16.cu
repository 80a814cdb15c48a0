// Decode kernel instantiations: cache PA_FP8_E4M3, q/out PA_F16 (one unit per dtype pair
// so the build compiles them in parallel).
#include "decode_launch.h"

namespace pa {
namespace dec {
cudaError_t launch_fp8_q_f16(const Launch& L) { return launch_dtype<PA_FP8_E4M3, PA_F16>(L); }
}  // namespace dec
}  // namespace pa
