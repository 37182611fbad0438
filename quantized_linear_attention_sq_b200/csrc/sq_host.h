// sq_host.h -- error reporting shared by the host sources of libsq.
#pragma once
#include <cuda_runtime.h>

#include <string>

#include "sq.h"

namespace sqi {

// Message of the last non-OK return on this host thread (sq_last_error).
extern thread_local std::string g_last_error;

// Record a printf-style message and return `s`.
sq_status fail(sq_status s, const char* fmt, ...);

// Record a CUDA runtime error and return SQ_ERR_CUDA.
sq_status cuda_fail(cudaError_t e, const char* what);

}  // namespace sqi
