// attn_tc05.cu -- tensor-core (tcgen05 / TMEM) step attention.  Not built yet.
#include "kernels.h"

namespace tidar {

cudaError_t launch_attn_tc05(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace tidar
