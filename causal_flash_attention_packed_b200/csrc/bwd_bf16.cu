#include "internal.h"
namespace fapk { cudaError_t launch_bwd_bf16(const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; } }
