// fa_bwd.cu - backward pass (placeholder until the sm_100a kernels land).
#include "fa_internal.h"

namespace fa {

fa_status launch_bwd(const void*, const void*, const void*, const void*, const void*,
                     const float*, void*, void*, void*, void*, int, int, int, int, int, float,
                     cudaStream_t) {
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
