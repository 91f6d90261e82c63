// rdr.cu -- rate-distortion retention (RDR) tier assignment and page-table
// construction.
//
// Spherical KV (arXiv 2605.18856), Abstract: RDR casts the allocation of KV
// storage as a rate-distortion trade-off, picking keep/drop and a precision
// tier together under a fixed budget, and the result is pages that each hold
// one tier with little metadata.  This library's reading:
// the unit is a 16-token page of one kv head; rate = page bytes of the tier,
// distortion = page utility x eps[tier]; a Lagrangian argmin with lambda found
// by doubling then 100 bisection steps, always keeping the feasible end.
//
// rdr_assign runs as ONE cooperative kernel (one CTA per SM, co-residency
// guaranteed by the cooperative launch): each evaluation of bytes(lambda) is a
// grid-wide int64 sum (exact, so independent of order), followed by a grid
// barrier after which every CTA takes the same decision.  The barrier spins on
// a global counter with an iteration limit; on expiry the kernel reports
// SPHKV_ERR_TIMEOUT and returns.
#include <cooperative_groups.h>

#include "common.cuh"

namespace sphkv {
namespace {

constexpr int kRdrThreads = 512;
constexpr long kSpinLimit = 1L << 24;

struct RdrParams {
    const int32_t* page_offsets;
    const int32_t* seq_lens;
    const float* utility;
    int64_t total_pages;
    int B, H_kv;
    double eps[4];
    double rate[4];
    int64_t budget;
    int n_sink, n_recent;
    uint8_t* tiers_out;
    const uint8_t* cap;        // re-run: current tiers, each unit may only get coarser (null: none)
    double* lambda_out;
    int64_t* bytes_out;
    int32_t* status;
    // workspace
    int32_t* seq_start;        // [B+1] prefix of token pages per sequence
    unsigned long long* acc;   // [3] rotating sums
    unsigned int* bar;         // grid barrier counter (zeroed before launch)
    int* abort_flag;
    double* U;                 // [n_units] page utility
    uint8_t* forced;           // [n_units]: bit 2 forced, bits 0..1 the finest allowed choice
};

// argmin over choices first..3 (T1, T2, T3, drop) of U eps + lambda R, ties to
// the lower index.
__device__ inline int choice(double U, const double* eps, const double* R, double lam, int first)
{
    int best = first;
    double bc = __dadd_rn(__dmul_rn(U, eps[first]), __dmul_rn(lam, R[first]));
    for (int t = first + 1; t < 4; ++t) {
        double c = __dadd_rn(__dmul_rn(U, eps[t]), __dmul_rn(lam, R[t]));
        if (c < bc) {
            bc = c;
            best = t;
        }
    }
    return best;
}

// Grid barrier number `gen` (1, 2, ...): arrive, then wait until every CTA has.
__device__ inline bool grid_barrier(const RdrParams& p, unsigned gen)
{
    __syncthreads();
    __shared__ int ok;
    if (threadIdx.x == 0) {
        ok = 1;
        __threadfence();
        atomicAdd(p.bar, 1u);
        const unsigned target = gen * gridDim.x;
        long i = 0;
        while (true) {
            unsigned v = *(volatile unsigned*)p.bar;
            if (v >= target) break;
            if (*(volatile int*)p.abort_flag) { ok = 0; break; }
            if (++i > kSpinLimit) {
                ok = 0;
                atomicExch(p.abort_flag, 1);
                report(p.status, SPHKV_ERR_TIMEOUT);
                break;
            }
            __nanosleep(100);
        }
        __threadfence();
    }
    __syncthreads();
    return ok != 0;
}

__device__ inline int64_t unit_entry(const RdrParams& p, int64_t pages_per_head, int64_t u, int32_t* pg_out,
                                     int32_t* np_out, int* b_out)
{
    const int g = (int)(u / pages_per_head);
    const int32_t x = (int32_t)(u % pages_per_head);
    int lo = 0, hi = p.B - 1;   // sequence holding page x
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.seq_start[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    *b_out = lo;
    *pg_out = x - p.seq_start[lo];
    *np_out = p.seq_start[lo + 1] - p.seq_start[lo];
    return (int64_t)g * p.total_pages + p.page_offsets[lo] + *pg_out;
}

__global__ void __launch_bounds__(kRdrThreads) rdr_kernel(RdrParams p)
{
    const int64_t pages_per_head = p.seq_start[p.B];
    const int64_t n_units = pages_per_head * p.H_kv;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    __shared__ unsigned long long red[kRdrThreads / 32];
    unsigned gen = 0;

    // Page utilities, summed once in slot order (fp64), and the forced flags.
    // The forced bytes are exact: every forced unit costs the page of the
    // finest tier it may take (T1 unless a re-run caps it).
    unsigned long long forced_mine = 0;
    for (int64_t u = gtid; u < n_units; u += stride) {
        int32_t pg, np;
        int b;
        const int64_t e = unit_entry(p, pages_per_head, u, &pg, &np, &b);
        const int len = p.seq_lens[b];
        const float* ut = p.utility + e * kP;
        double s = 0.0;
        for (int k = 0; k < kP && pg * kP + k < len; ++k) s = __dadd_rn(s, (double)ut[k]);
        const bool forced = pg < p.n_sink || pg >= np - p.n_recent;
        int first = 0;   // a re-run may only make a unit coarser
        if (p.cap) {
            const int ct = p.cap[e];
            first = ct == 0 ? 3 : (ct <= 3 ? ct - 1 : 3);
        }
        p.U[u] = s;
        p.forced[u] = (uint8_t)((forced ? 4 : 0) | first);
        if (forced) forced_mine += (unsigned long long)p.rate[first];
    }
    // Block-sum `mine` into acc[slot], then a grid barrier.
    auto commit = [&](unsigned long long mine, int slot) -> bool {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mine;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long t = 0;
            for (int w = 0; w < kRdrThreads / 32; ++w) t += red[w];
            atomicAdd(p.acc + slot, t);
            if (blockIdx.x == 0) p.acc[(slot + 1) % 3] = 0ull;   // unread since two barriers
        }
        return grid_barrier(p, ++gen);
    };
    auto eval = [&](double lam, int slot) -> bool {   // bytes(lam) into acc[slot]
        unsigned long long mine = 0;
        for (int64_t u = gtid; u < n_units; u += stride)
        {
            const int f = p.forced[u], first = f & 3;
            mine += (unsigned long long)((f & 4) ? p.rate[first] : p.rate[choice(p.U[u], p.eps, p.rate, lam, first)]);
        }
        return commit(mine, slot);
    };
    auto total = [&](int slot) -> int64_t { return (int64_t)(*(volatile unsigned long long*)(p.acc + slot)); };

    int it = 0;
    if (!commit(forced_mine, it % 3)) return;
    const int64_t forced_bytes = total(it % 3);
    ++it;
    if (forced_bytes > p.budget) {
        if (gtid == 0) report(p.status, SPHKV_ERR_BUDGET);
        return;
    }
    double lo = 0.0, hi = 1.0;
    if (!eval(hi, it % 3)) return;
    int64_t bh = total(it % 3);
    ++it;
    for (int k = 0; k < 2000 && bh > p.budget; ++k) {
        hi = __dmul_rn(hi, 2.0);
        if (!eval(hi, it % 3)) return;
        bh = total(it % 3);
        ++it;
    }
    for (int step = 0; step < 100; ++step) {
        const double mid = __dadd_rn(lo, __dmul_rn(__dadd_rn(hi, -lo), 0.5));
        if (!eval(mid, it % 3)) return;
        const int64_t bm = total(it % 3);
        ++it;
        if (bm <= p.budget) hi = mid;
        else lo = mid;
    }
    if (!eval(hi, it % 3)) return;
    bh = total(it % 3);
    for (int64_t u = gtid; u < n_units; u += stride) {
        int32_t pg, np;
        int b;
        const int64_t e = unit_entry(p, pages_per_head, u, &pg, &np, &b);
        const int f = p.forced[u], first = f & 3;
        const int t = (f & 4) ? first : choice(p.U[u], p.eps, p.rate, hi, first);
        p.tiers_out[e] = (uint8_t)(t == 3 ? 0 : t + 1);
    }
    if (gtid == 0) {
        *p.lambda_out = hi;
        *p.bytes_out = bh;
    }
}

// seq_start[b] = pages holding tokens before sequence b (ceil(len/16) each).
__global__ void __launch_bounds__(1024) seq_scan_kernel(const int32_t* seq_lens, const int32_t* page_offsets,
                                                        int B, int64_t total_pages, int32_t* seq_start,
                                                        int32_t* status)
{
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < B; base += 1024) {
        const int b = base + tid;
        int32_t n = 0;
        if (b < B) {
            const int64_t len = seq_lens[b];
            int64_t np = (len + kP - 1) / kP;
            const int64_t first = page_offsets[b], last = page_offsets[b + 1];
            int64_t cap = last - first;
            if (first < 0 || cap < 0 || last > total_pages) {   // inconsistent descriptor
                report(status, SPHKV_ERR_DATA);
                cap = 0;
            }
            if (len < 0 || np > cap) {
                report(status, SPHKV_ERR_DATA);
                np = len < 0 ? 0 : cap;
            }
            n = (int32_t)np;
        }
        int32_t x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int32_t t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        const int32_t excl = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - n;
        if (b < B) seq_start[b] = excl;
        __syncthreads();
        if (tid == 1023) carry = excl + n;
        __syncthreads();
    }
    if (tid == 0) seq_start[B] = carry;
}

// --------------------------------------------------------- page table --
__global__ void __launch_bounds__(1024) page_table_kernel(const uint8_t* tiers, int64_t n, const int32_t* perm1,
                                                          const int32_t* perm2, const int32_t* perm3,
                                                          int32_t* table, int64_t* counts, int32_t* status)
{
    __shared__ int64_t warp_tot[3][32];
    __shared__ int64_t carry[3];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid < 3) carry[tid] = 0;
    __syncthreads();
    const int32_t* perm[4] = {nullptr, perm1, perm2, perm3};
    for (int64_t base = 0; base < n; base += 1024) {
        const int64_t i = base + tid;
        int t = i < n ? tiers[i] : 0;
        if (t > 3) {
            report(status, SPHKV_ERR_DATA);
            t = 0;
        }
        int64_t x[3];
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            x[k] = (t == k + 1) ? 1 : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, x[k], o);
                if (lane >= o) x[k] += y;
            }
            if (lane == 31) warp_tot[k][w] = x[k];
        }
        __syncthreads();
        if (w < 3) {
            int64_t v = warp_tot[w][lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += y;
            }
            warp_tot[w][lane] = v;
        }
        __syncthreads();
        if (i < n) {
            if (t == 0) {
                table[i] = 0;
            } else {
                const int k = t - 1;
                const int64_t rank = carry[k] + (w > 0 ? warp_tot[k][w - 1] : 0) + x[k] - 1;
                const int64_t phys = perm[t] ? perm[t][rank] : rank;
                table[i] = (int32_t)(((uint32_t)t << 30) | ((uint32_t)phys & 0x3fffffffu));
            }
        }
        __syncthreads();
        if (tid < 3) carry[tid] += warp_tot[tid][31];
        __syncthreads();
    }
    if (tid < 3 && counts) counts[tid] = carry[tid];
}

size_t rdr_ws_layout(int B, int H_kv, int64_t total_pages, size_t* acc_off, size_t* bar_off, size_t* u_off,
                     size_t* f_off)
{
    const size_t n_units = (size_t)H_kv * (size_t)total_pages;
    size_t off = ((size_t)(B + 1) * 4 + 255) / 256 * 256;
    *acc_off = off;
    off += 256;
    *bar_off = off;
    off += 256;
    *u_off = off;
    off += (n_units * 8 + 255) / 256 * 256;
    *f_off = off;
    off += (n_units + 255) / 256 * 256;
    return off;
}

}  // namespace
}  // namespace sphkv

using namespace sphkv;

extern "C" size_t sphkv_rdr_workspace_bytes(int32_t B, int32_t H_kv, int64_t total_pages)
{
    if (B <= 0 || H_kv <= 0 || total_pages < 0) return 0;
    size_t a, b, u, f;
    return rdr_ws_layout(B, H_kv, total_pages, &a, &b, &u, &f);
}

namespace {
sphkv_status rdr_launch(const char* fn, bool rerun, const sphkv_cache* c, const float* utility, const double* eps,
                        int64_t budget_bytes, int32_t n_sink, int32_t n_recent, uint8_t* tiers_out,
                        double* lambda_out, int64_t* bytes_out, void* workspace, size_t ws_bytes,
                        int32_t* status_dev, void* stream);
}

extern "C" sphkv_status sphkv_rdr_assign(const sphkv_cache* c, const float* utility, const double* eps,
                                         int64_t budget_bytes, int32_t n_sink, int32_t n_recent,
                                         uint8_t* tiers_out, double* lambda_out, int64_t* bytes_out,
                                         void* workspace, size_t ws_bytes, int32_t* status_dev,
                                         void* stream)
{
    const CallRange range("sphkv_rdr_assign");
    return rdr_launch("sphkv_rdr_assign", false, c, utility, eps, budget_bytes, n_sink, n_recent, tiers_out,
                      lambda_out, bytes_out, workspace, ws_bytes, status_dev, stream);
}

extern "C" sphkv_status sphkv_rdr_rerun(const sphkv_cache* c, const float* utility, const double* eps,
                                        int64_t budget_bytes, int32_t n_sink, int32_t n_recent, uint8_t* tiers_io,
                                        double* lambda_out, int64_t* bytes_out, void* workspace, size_t ws_bytes,
                                        int32_t* status_dev, void* stream)
{
    const CallRange range("sphkv_rdr_rerun");
    return rdr_launch("sphkv_rdr_rerun", true, c, utility, eps, budget_bytes, n_sink, n_recent, tiers_io,
                      lambda_out, bytes_out, workspace, ws_bytes, status_dev, stream);
}

namespace {
sphkv_status rdr_launch(const char* fn, bool rerun, const sphkv_cache* c, const float* utility, const double* eps,
                        int64_t budget_bytes, int32_t n_sink, int32_t n_recent, uint8_t* tiers_out,
                        double* lambda_out, int64_t* bytes_out, void* workspace, size_t ws_bytes,
                        int32_t* status_dev, void* stream)
{
    if (!c || !utility || !eps || !tiers_out || !lambda_out || !bytes_out || !workspace) {
        sphkv_set_error("%s: null argument", fn);
        return SPHKV_ERR_ARG;
    }
    if (c->B <= 0 || c->H_kv <= 0 || !c->page_offsets || !c->seq_lens || c->total_pages < 0) {
        sphkv_set_error("%s: bad cache descriptor", fn);
        return SPHKV_ERR_ARG;
    }
    if (n_sink < 0 || n_recent < 0 || budget_bytes < 0) {
        sphkv_set_error("%s: n_sink, n_recent and budget must be >= 0", fn);
        return SPHKV_ERR_ARG;
    }
    if ((int64_t)c->H_kv * c->total_pages > 0x7fffffffLL) {
        sphkv_set_error("%s: cache too large for 32-bit page indices", fn);
        return SPHKV_ERR_ARG;
    }
    size_t acc_off, bar_off, u_off, f_off;
    const size_t need = rdr_ws_layout(c->B, c->H_kv, c->total_pages, &acc_off, &bar_off, &u_off, &f_off);
    if (ws_bytes < need || ((uintptr_t)workspace & 255)) {
        sphkv_set_error("%s: workspace must be 256-byte aligned and >= %zu bytes", fn, need);
        return SPHKV_ERR_ARG;
    }
    RdrParams p{};
    p.page_offsets = c->page_offsets;
    p.seq_lens = c->seq_lens;
    p.utility = utility;
    p.total_pages = c->total_pages;
    p.B = c->B;
    p.H_kv = c->H_kv;
    for (int t = 0; t < 4; ++t) p.eps[t] = eps[t];
    for (int t = 0; t < 3; ++t) p.rate[t] = (double)page_bytes_of(t + 1);
    p.rate[3] = 0.0;
    p.budget = budget_bytes;
    p.n_sink = n_sink;
    p.n_recent = n_recent;
    p.tiers_out = tiers_out;
    p.cap = rerun ? tiers_out : nullptr;   // read per unit before the same unit's write
    p.lambda_out = lambda_out;
    p.bytes_out = bytes_out;
    p.status = status_dev;
    uint8_t* ws = (uint8_t*)workspace;
    p.seq_start = (int32_t*)ws;
    p.acc = (unsigned long long*)(ws + acc_off);
    p.bar = (unsigned int*)(ws + bar_off);
    p.abort_flag = (int*)(ws + bar_off + 4);
    p.U = (double*)(ws + u_off);
    p.forced = ws + f_off;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(ws + acc_off, 0, 512, s) != cudaSuccess) {
        sphkv_set_error("%s: memset failed", fn);
        return SPHKV_ERR_DEVICE;
    }
    seq_scan_kernel<<<1, 1024, 0, s>>>(c->seq_lens, c->page_offsets, c->B, c->total_pages, p.seq_start,
                                       status_dev);
    int dev = 0, n_sm = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rdr_kernel, kRdrThreads, 0);
    if (per_sm < 1 || n_sm < 1) {
        sphkv_set_error("%s: no cooperative occupancy", fn);
        return SPHKV_ERR_DEVICE;
    }
    void* args[] = {&p};
    cudaError_t err = cudaLaunchCooperativeKernel((const void*)rdr_kernel, dim3(n_sm), dim3(kRdrThreads),
                                                  args, 0, s);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("%s: launch failed: %s", fn, cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}
}  // namespace

extern "C" sphkv_status sphkv_build_page_table(const uint8_t* tiers, int64_t n_entries, const int32_t* perm1,
                                               const int32_t* perm2, const int32_t* perm3, int32_t* table,
                                               int64_t* counts_out, int32_t* status_dev, void* stream)
{
    const CallRange range("sphkv_build_page_table");
    if (n_entries < 0 || (n_entries > 0 && (!tiers || !table))) {
        sphkv_set_error("sphkv_build_page_table: bad arguments");
        return SPHKV_ERR_ARG;
    }
    page_table_kernel<<<1, 1024, 0, (cudaStream_t)stream>>>(tiers, n_entries, perm1, perm2, perm3, table,
                                                           counts_out, status_dev);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("sphkv_build_page_table: launch failed: %s", cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}
