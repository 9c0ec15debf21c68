// fa_bwd_sm100.cu -- BF16 attention backward for sm_100a (placeholder until
// the tcgen05 dK/dV kernel lands).
#include "common.cuh"
#include "launch.h"

namespace fa {
int launch_bwd_bf16_sm100(const AttnArgs &) { return 2; }
}  // namespace fa
