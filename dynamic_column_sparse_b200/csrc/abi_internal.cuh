// abi_internal.cuh - helpers of the C ABI implementation shared between its
// translation units (api.cu defines them).
#pragma once

#include <cuda_runtime.h>

#include "../../include/chipmunk.h"

namespace cm {

// Records `msg` for chipmunk_last_error (this host thread) and returns st.
chipmunk_status record_error(chipmunk_status st, const char *msg);

// chipmunk_mlp_delta with its delta scratch taken from get_scratch instead of
// a caller workspace. The arguments are checked first; a step that needs more
// than scratch_bytes is rejected with CHIPMUNK_ERR_WORKSPACE before anything
// else happens. get_scratch runs after the device checks, with the caller's
// device current.
chipmunk_status mlp_delta_fixed_scratch(const chipmunk_mlp_args *a, size_t scratch_bytes,
                                        chipmunk_status (*get_scratch)(void **), cudaStream_t s);

}  // namespace cm
