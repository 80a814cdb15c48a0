// Host-side internals shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "pa.h"

namespace pa {

// Record a failure for pa_last_error() on this thread and return the status.
pa_status fail(pa_status st, const char* fmt, ...);
void clear_error();

inline int elem_size(pa_dtype dt) {
    switch (dt) {
    case PA_F32: return 4;
    case PA_F16: case PA_BF16: return 2;
    case PA_FP8_E4M3: return 1;
    }
    return 0;
}

inline bool valid_dtype(int dt) { return dt >= PA_F32 && dt <= PA_FP8_E4M3; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the sticky error word of the current device (nullptr and
// a recorded error if the runtime call fails).
unsigned int* device_error_word();

// Translate a CUDA runtime error into PA_ERR_CUDA with context.
pa_status cuda_fail(int err, const char* what);

}  // namespace pa
