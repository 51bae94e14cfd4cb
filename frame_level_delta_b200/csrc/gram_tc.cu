// Frame statistics on tcgen05 tensor cores (bf16 operands, fp32 accumulation in TMEM).
#include "internal.h"

namespace vda {

bool gram_tc_supported(const Problem& p) { return false; }
cudaError_t launch_gram_tc(const Problem& p, cudaStream_t s) { return cudaErrorNotSupported; }

}  // namespace vda
