// Decode kernel instantiations: cache PA_BF16, q/out PA_BF16 (one unit per dtype pair
// so the build compiles them in parallel).
#include "decode_launch.h"

namespace pa {
namespace dec {
cudaError_t launch_bf16(const Launch& L) { return launch_dtype<PA_BF16, PA_BF16>(L); }
}  // namespace dec
}  // namespace pa
