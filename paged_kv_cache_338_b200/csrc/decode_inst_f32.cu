// Decode kernel instantiations: cache PA_F32, q/out PA_F32 (one unit per dtype pair
// so the build compiles them in parallel).
#include "decode_launch.h"

namespace pa {
namespace dec {
cudaError_t launch_f32(const Launch& L) { return launch_dtype<PA_F32, PA_F32>(L); }
}  // namespace dec
}  // namespace pa
