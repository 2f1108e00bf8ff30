// Thread-local error message behind pa_last_error().
#pragma once

#include <cstdarg>
#include <cstdio>

namespace pa {

char *error_buffer();  // thread-local, 512 bytes

inline void clear_error() { error_buffer()[0] = '\0'; }

inline int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(error_buffer(), 512, fmt, ap);
    va_end(ap);
    return code;
}

}  // namespace pa
