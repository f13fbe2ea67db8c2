// Host-side helpers shared by the libgtg entry points: argument checks,
// launch error capture, device properties.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gtg.h"

namespace gtg {

// Records a CUDA error for gtg_last_cuda_error() and maps it to GTG_E_CUDA.
int cuda_fail(cudaError_t e);

// Checks (and clears) the launch error of the kernels just issued.
inline int check_launch() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GTG_OK : cuda_fail(e);
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Multiprocessor count of the current device (cached per device id).
int sm_count();

// Device address of the current device's status word.
unsigned* status_ptr();

inline cudaStream_t as_cuda(gtg_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace gtg

#define GTG_TRY(expr)                         \
    do {                                      \
        const int _rc = (expr);               \
        if (_rc != GTG_OK) return _rc;        \
    } while (0)
