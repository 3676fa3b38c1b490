// bf16 attention forward on the 5th-generation tensor cores (tcgen05 / TMEM).
#include "internal.h"

namespace gqa {

int launch_fwd_bf16(const FwdTensors&, const FwdParams&, cudaStream_t) { return GQA_ERR_UNSUPPORTED; }

}  // namespace gqa
