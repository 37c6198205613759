// S3 on the 5th-generation tensor cores (tcgen05, TMEM, TMA): placeholder
// until the kernel lands; mla_decode falls back to the CUDA-core kernel.
#include "mla_internal.cuh"

namespace mla {

bool decode_tc_supported(const mla_dims&, int) { return false; }

int decode_tc_auto_splits(int num_sms, int n_q) { return num_sms / 2 / (n_q > 0 ? n_q : 1); }

cudaError_t launch_decode_tc(const DecodeParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mla
