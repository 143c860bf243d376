// Argument checks of the C ABI shared by the entry points in moe_abi.cu and
// permute_no_alloc.cu (internal to the library).
#pragma once

#include "launch.h"
#include "moe.h"

namespace moe {

// moe_shape_t -> Dims with every rule of include/moe.h (sizes, dtype, alignment multiples,
// gate mode, expert format); MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED otherwise.
moe_status_t to_dims(const moe_shape_t* s, Dims* D);
// The current device is an sm_100 part (MOE_ERR_UNSUPPORTED otherwise, MOE_ERR_CUDA when the
// runtime cannot tell).
moe_status_t check_device();
moe_status_t check_ws(const Dims& D, void* ws, size_t ws_bytes);

}  // namespace moe
