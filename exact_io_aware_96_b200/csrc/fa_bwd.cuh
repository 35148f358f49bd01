// fa_bwd.cuh — attention backward for sm_100a (placeholder until the kernels land).
#pragma once

#include "fa.h"
#include "fa_common.cuh"

namespace fa {

inline int launch_bwd(const fa_bwd_params*, cudaStream_t) { return FA_ERR_NOT_IMPLEMENTED; }

}  // namespace fa
