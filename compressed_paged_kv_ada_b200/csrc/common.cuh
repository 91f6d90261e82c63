// common.cuh -- format constants and device helpers shared by the libsphkv
// kernels (encode, RDR, page table, decode).  Nothing here is used by, or
// uses, the CPU oracle.
//
// Page format (Spherical KV, arXiv 2605.18856, Abstract: every page holds
// one tier, carries little metadata and is read contiguously; the byte layout
// is this library's, described in include/sphkv.h):
//   r[16] fp16 | vscale[16] fp16 | code planes (8 subtree blocks per token)
//   | value rows (channels permuted for tensor-core fragments)
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "../../include/sphkv.h"

namespace sphkv {

// A named NVTX range around one C-ABI call, so that timeline tools (nsys, ncu's
// range filters) can attribute the call's launches; without a tool attached
// it costs a load and a branch.
struct CallRange {
    explicit CallRange(const char* name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange&) = delete;
    CallRange& operator=(const CallRange&) = delete;
};

constexpr int kD = SPHKV_HEAD_DIM;      // 128
constexpr int kP = SPHKV_PAGE_TOKENS;   // 16
constexpr int kLeaves = kD / 2;         // 64
constexpr int kUpper = kD / 2 - 1;      // 63

struct TierFmt {
    int b_leaf, b_up, v_bits;
    int code_row;     // code bytes per token (8 subtree blocks)
    int v_row;        // value bytes per token
    int off_codes, off_v;
    int page_bytes;
};

__host__ __device__ constexpr TierFmt make_fmt(int bl, int bu, int vb, int code_row)
{
    return TierFmt{bl, bu, vb, code_row, kD * vb / 8, 4 * kP, 4 * kP + kP * code_row,
                   4 * kP + kP * code_row + kP * (kD * vb / 8)};
}

// Tier index 1..3 (0 = drop).
template <int T>
struct Tier;
template <>
struct Tier<1> { static constexpr TierFmt f = make_fmt(8, 8, 8, 128); };
template <>
struct Tier<2> { static constexpr TierFmt f = make_fmt(4, 6, 4, 80); };
template <>
struct Tier<3> { static constexpr TierFmt f = make_fmt(3, 4, 4, 56); };

static_assert(Tier<1>::f.page_bytes == 4160, "T1 page");
static_assert(Tier<2>::f.page_bytes == 2368, "T2 page");
static_assert(Tier<3>::f.page_bytes == 1984, "T3 page");
static_assert(Tier<1>::f.page_bytes % 16 == 0 && Tier<2>::f.page_bytes % 16 == 0 &&
                  Tier<3>::f.page_bytes % 16 == 0,
              "pages must be 16-byte multiples for bulk copies");

// Value row position p = 16g + 2m + h holds channel 16m + g + 8h.
__host__ __device__ constexpr int v_channel_at(int p) { return 16 * ((p >> 1) & 7) + (p >> 4) + 8 * (p & 1); }

__host__ __device__ inline int page_bytes_of(int t)
{
    return t == 1 ? Tier<1>::f.page_bytes
                  : t == 2 ? Tier<2>::f.page_bytes : t == 3 ? Tier<3>::f.page_bytes : 0;
}

// Page-table entry: bits 31..30 tier, 29..0 pool page.
__host__ __device__ inline int entry_tier(int32_t e) { return (int)(((uint32_t)e) >> 30); }
__host__ __device__ inline int64_t entry_page(int32_t e) { return (int64_t)(((uint32_t)e) & 0x3fffffffu); }

// Record a device-side error: the largest code wins, so the result does not
// depend on the order in which threads report.
__device__ inline void report(int32_t* status, int code)
{
    if (status) atomicMax(status, code);
}

}  // namespace sphkv

// Host-side error text (per thread), set by the entry points.
void sphkv_set_error(const char* fmt, ...);
