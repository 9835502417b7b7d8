// k_prefill_tc.cu -- tcgen05 / TMEM pre-fill attention (bf16, head_dim 128).
#include "device_common.cuh"

namespace duo {

bool prefill_tc_supported(const PrefillParams &, duo_dtype) { return false; }

cudaError_t launch_prefill_tc(const PrefillParams &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace duo
