// fa_internal.h -- checks shared by the library's translation units (not part
// of the C ABI; hidden symbols).
#pragma once

#include "fa.h"

namespace fa_detail {

// Every argument check of fa_fwd_ex that needs no device, except the
// caller-owned workspace clause (which fa_fwd_static_workspace replaces).
fa_status validate_args(const fa_fwd_params *p);

// FA_OK when the current device is an sm_100 device the library supports
// (cached per device ordinal); FA_ERR_UNSUPPORTED or FA_ERR_CUDA otherwise.
fa_status probe_current_device();

}  // namespace fa_detail
