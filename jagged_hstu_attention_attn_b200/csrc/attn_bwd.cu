// attn_bwd.cu -- backward (placeholder until the kernel lands)
#include "internal.h"
namespace hstu {
cudaError_t attn_bwd_launch(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}
