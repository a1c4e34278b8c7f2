// Tensor-core (tcgen05) decode path for grouped query heads.
#include "decode_common.cuh"
#include "pkv_internal.h"

namespace pkv {

bool tensor_path_supports(int group, int head_dim) { return false; }

int launch_decode_tensor(const DecodeArgs&, int, bool, cudaStream_t) {
  return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: tensor path not available");
}

}  // namespace pkv
