// keep.cu -- per-token keep/drop inside kept pages.
//
// Spherical KV (arXiv 2605.18856), Abstract: RDR decides keep/drop per token
// and head.  A stored radius is fp16(|k|) >= +0, so its sign bit is free: it
// is the token's drop flag (1 = dropped) and the decode skips such a token
// exactly as if it were absent.  Pages stay tier-homogeneous and their size
// does not change.
#include "common.cuh"

namespace sphkv {
namespace {

struct KeepParams {
    const int32_t* page_offsets;
    const int32_t* seq_lens;
    const int32_t* page_table;
    uint8_t* pool[4];
    int64_t pool_pages[4];
    int64_t total_pages;
    int B, H_kv;
    const uint8_t* keep;   // [H_kv][total_pages * 16]
    int32_t* status;
};

// Sequence owning logical page lp: the last b with page_offsets[b] <= lp.
__device__ inline int seq_of_page(const int32_t* po, int B, int64_t lp)
{
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (po[mid] <= lp) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// One thread per (kv head, logical page, slot); each writes only its own
// token's radius, so no two threads touch the same bytes.
__global__ void set_keep_kernel(KeepParams p)
{
    const int64_t per_head = p.total_pages * kP;
    const int64_t n = per_head * p.H_kv;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int g = (int)(i / per_head);
        const int64_t lp = (i % per_head) / kP;
        const int slot = (int)(i % kP);
        const int b = seq_of_page(p.page_offsets, p.B, lp);
        if (lp >= p.page_offsets[b + 1]) continue;   // a page past the last sequence
        const int64_t pos = (lp - p.page_offsets[b]) * kP + slot;
        if (pos >= p.seq_lens[b]) continue;          // no token in this slot
        const int32_t e = p.page_table[(int64_t)g * p.total_pages + lp];
        const int t = entry_tier(e);
        if (t == 0) continue;
        if (entry_page(e) >= p.pool_pages[t]) {
            report(p.status, SPHKV_ERR_DATA);
            continue;
        }
        uint16_t* r = (uint16_t*)(p.pool[t] + entry_page(e) * (int64_t)page_bytes_of(t)) + slot;
        *r = p.keep[i] ? (uint16_t)(*r & 0x7fffu) : (uint16_t)(*r | 0x8000u);
    }
}

}  // namespace
}  // namespace sphkv

using namespace sphkv;

extern "C" sphkv_status sphkv_set_keep(const sphkv_cache* c, const uint8_t* keep, int32_t* status_dev, void* stream)
{
    const char* fn = "sphkv_set_keep";
    const CallRange range(fn);
    if (!c || !keep) {
        sphkv_set_error("%s: null argument", fn);
        return SPHKV_ERR_ARG;
    }
    if (c->B <= 0 || c->H_kv <= 0 || c->total_pages < 0 || !c->page_offsets || !c->seq_lens || !c->page_table) {
        sphkv_set_error("%s: bad cache descriptor", fn);
        return SPHKV_ERR_ARG;
    }
    if (c->total_pages == 0) return SPHKV_OK;
    KeepParams p{};
    p.page_offsets = c->page_offsets;
    p.seq_lens = c->seq_lens;
    p.page_table = c->page_table;
    for (int t = 1; t <= 3; ++t) {
        p.pool[t] = c->pool[t - 1];
        p.pool_pages[t] = c->pool[t - 1] ? c->pool_pages[t - 1] : 0;
    }
    p.total_pages = c->total_pages;
    p.B = c->B;
    p.H_kv = c->H_kv;
    p.keep = keep;
    p.status = status_dev;
    const int64_t n = c->total_pages * kP * c->H_kv;
    const int64_t blocks = (n + 255) / 256 < 148 * 32 ? (n + 255) / 256 : 148 * 32;
    set_keep_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(p);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("%s: launch failed: %s", fn, cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}
