// Internal helpers shared by the translation units of libpa_b200.so.
#pragma once

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "pa.h"

namespace pa {

// Records a printf-style message as this thread's last error and returns `st`.
pa_status fail(pa_status st, const char* fmt, ...);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int dtype_bytes(pa_dtype dt) {
  switch (dt) {
    case PA_F32: return 4;
    case PA_BF16: return 2;
    case PA_F16: return 2;
  }
  return 0;
}

}  // namespace pa
