// api.cu -- host-side helpers of the libsphkv C ABI: per-thread error text and
// the page sizes of the tier format.
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace {
thread_local char g_err[512] = "";
}

void sphkv_set_error(const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

extern "C" const char* sphkv_last_error(void) { return g_err; }

extern "C" int sphkv_page_bytes(int tier) { return sphkv::page_bytes_of(tier); }
