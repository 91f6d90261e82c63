// decode.cu -- angle-domain attention (ADA) decode over the paged cache.
//
// Spherical KV (arXiv 2605.18856), Abstract: logits come "directly from these
// codes without reconstructing dense keys", on "a paged, block-local,
// fusion-friendly decode path" that "directly targets HBM traffic".  The logit
// of query q against a stored key is r * S_root / sqrt(d), with S evaluated
// bottom-up over the recursive-polar tree:
//   leaf j:     S = q[2j] cos(phi_j) + q[2j+1] sin(phi_j)
//   upper node: S = cos(psi) S_left + sin(psi) S_right.
// Values are dequantised (int8/int4 code times the token's fp16 scale) inside
// the value FMA; an online softmax keeps (max, sum, out) per query head, and
// long contexts are split across SMs and merged with a log-sum-exp combine.
//
// Launch structure (three kernels on the caller's stream):
//   plan   -- 1 CTA: unit_start[u] = pages before unit u = (b, g), u = b*H_kv+g.
//   decode -- persistent, one 512-thread CTA per SM.  The flattened page range
//             [0, P) is cut into n_cta equal pieces; a CTA walks the units its
//             piece overlaps.  Its 16 warps take the unit's pages round robin;
//             each warp bulk-copies a page (cp.async.bulk, mbarrier completion)
//             into a 2-stage ring in shared memory while it computes the
//             previous one.  A warp covers 4 tokens per pass, 8 lanes per
//             token, each lane an 8-leaf subtree; the three top tree levels
//             use shuffles that hand each lane a different query head.  The
//             per-tier cos/sin tables sit in shared memory, replicated 16
//             times so a half-warp's 64-bit lookups never share a bank.
//   merge  -- one CTA per unit whose pages were split over several CTAs.
#include "common.cuh"

namespace sphkv {
namespace {

constexpr int kG = 4;               // query heads per kv head
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 2;
constexpr int kStageBytes = Tier<1>::f.page_bytes;  // largest page
constexpr int kRep = 16;            // LUT replicas (one per lane of a half warp)
constexpr int kMinPagesPerCta = 64;
constexpr int kPartStride = 132;    // floats per (slot, head): m, l, pad, pad, o[128]

// LUT entries: leaf tables of T1/T2/T3 then upper tables of T1/T2/T3.
constexpr int kLeafBase1 = 0, kLeafBase2 = 256, kLeafBase3 = 272;
constexpr int kUpBase1 = 280, kUpBase2 = 536, kUpBase3 = 600;
constexpr int kLutEntries = 616;

constexpr int kLutBytes = kLutEntries * kRep * 8;
constexpr int kStageOff = kLutBytes;
constexpr int kPbufOff = kStageOff + kWarps * kStages * kStageBytes;
constexpr int kPbufFloats = 16 * kG + kG;   // p*scale per (token, head), then alpha per head
constexpr int kBarOff = kPbufOff + kWarps * kPbufFloats * 4;
constexpr int kSmemBytes = kBarOff + kWarps * kStages * 8;
static_assert(kStageOff % 128 == 0 && kPbufOff % 16 == 0 && kBarOff % 8 == 0, "smem alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
// CTA merge scratch (aliases the stage ring): m[16][4], l[16][4], o[16][4][128]
static_assert((2 * kWarps * kG + kWarps * kG * kD) * 4 <= kWarps * kStages * kStageBytes, "merge scratch");

constexpr float kLn2 = 0.6931471805599453f;
// log2(e) / sqrt(128): logits are kept in the log2 domain
constexpr float kLogitScale = 0.12751743082459868f;

constexpr long kWaitLimit = 1L << 22;

template <int T>
struct TierLut;
template <>
struct TierLut<1> { static constexpr int leaf = kLeafBase1, up = kUpBase1; };
template <>
struct TierLut<2> { static constexpr int leaf = kLeafBase2, up = kUpBase2; };
template <>
struct TierLut<3> { static constexpr int leaf = kLeafBase3, up = kUpBase3; };

struct DecodeParams {
    const int32_t* page_offsets;
    const int32_t* seq_lens;
    const int32_t* page_table;
    const uint8_t* pool[4];
    int64_t pool_pages[4];
    int64_t total_pages;
    int B, H_kv, H_q, n_units, n_cta;
    const float* q;
    float* out;
    float* lse;
    int32_t* unit_start;   // [n_units + 1]
    float* partial;        // [n_cta + n_units][kG][kPartStride]
    int32_t* status;
};

// ------------------------------------------------------------- PTX glue --
__device__ inline uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ inline void mbar_init(uint32_t bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ inline void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ inline void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ inline void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ inline bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase; false if the limit ran out.
__device__ inline bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (long i = 0; i < kWaitLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (i > 16) __nanosleep(64);
    }
    return false;
}

__device__ inline uint32_t ld_u32(const uint8_t* p) { return *(const uint32_t*)p; }

// 32 bits of a row's LSB-first bit stream starting at bit `pos` (row 4-byte aligned).
__device__ inline uint32_t bits_at(const uint8_t* row, int pos)
{
    const uint32_t* w = (const uint32_t*)row + (pos >> 5);
    return __funnelshift_r(w[0], w[1], pos & 31);
}

// ---------------------------------------------------------------- plan --
__global__ void __launch_bounds__(1024) plan_kernel(DecodeParams p)
{
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < p.n_units; base += 1024) {
        int u = base + tid;
        int32_t n = 0;
        if (u < p.n_units) {
            int b = u / p.H_kv;
            const int64_t first = p.page_offsets[b], last = p.page_offsets[b + 1];
            int64_t cap = last - first;
            if (first < 0 || cap < 0 || last > p.total_pages) {   // inconsistent descriptor
                report(p.status, SPHKV_ERR_DATA);
                cap = 0;
            }
            int64_t len = p.seq_lens[b];
            int64_t np = (len + kP - 1) / kP;
            if (len < 0 || np > cap) {
                report(p.status, SPHKV_ERR_DATA);
                np = len < 0 ? 0 : cap;
            }
            n = (int32_t)np;
        }
        int32_t x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int32_t t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        int32_t excl = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - n;
        if (u < p.n_units) p.unit_start[u] = excl;
        __syncthreads();
        if (tid == 1023) carry = excl + n;
        __syncthreads();
    }
    if (tid == 0) p.unit_start[p.n_units] = carry;
}

// Largest u in [0, n_units) with unit_start[u] <= x < unit_start[u+1].
__device__ inline int find_unit(const int32_t* us, int n_units, int32_t x)
{
    int lo = 0, hi = n_units - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (us[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ inline int32_t cta_bound(int c, int32_t P, int n_cta)
{
    return (int32_t)(((int64_t)c * P) / n_cta);
}

// ------------------------------------------------------------- page work --
struct WarpState {
    float m;        // running max (log2 domain) of this lane's head
    float l;        // running sum of this lane's tokens
    float o[kG][4]; // out accumulators: 4 heads x dims 4*lane .. 4*lane+3
};

__device__ inline float2 lut_get(const float2* lut, int entry, int lane)
{
    return lut[entry * kRep + (lane & (kRep - 1))];
}

// One page of tier T already staged in shared memory at `pg`.
template <int T>
__device__ __forceinline__ void process_page(const uint8_t* pg, int valid, const float (&qr)[kG][16],
                                             const float2* lut, float* pbuf, int lane,
                                             WarpState& st)
{
    constexpr TierFmt F = Tier<T>::f;
    constexpr int LB = TierLut<T>::leaf, UB = TierLut<T>::up;
    constexpr uint32_t LM = (1u << F.b_leaf) - 1, UM = (1u << F.b_up) - 1;
    const unsigned full = 0xffffffffu;
    const int k = lane >> 3, s = lane & 7;
    const int head = (s & 1) * 2 + ((s >> 1) & 1);   // head held after the shuffle levels
    float lg[4];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int t = pass * 4 + k;
        const uint8_t* lrow = pg + F.off_leaf + t * F.leaf_row;
        const uint8_t* urow = pg + F.off_up + t * F.up_row;
        // leaf codes of leaves 8s .. 8s+7
        uint32_t lc0, lc1 = 0;
        if (F.b_leaf == 8) {
            lc0 = ld_u32(lrow + 8 * s);
            lc1 = ld_u32(lrow + 8 * s + 4);
        } else if (F.b_leaf == 4) {
            lc0 = ld_u32(lrow + 4 * s);
        } else {
            lc0 = bits_at(lrow, 8 * s * F.b_leaf);
        }
        const uint32_t u1 = bits_at(urow, (4 * s) * F.b_up);          // level 1: nodes 4s..4s+3
        const uint32_t u2 = bits_at(urow, (32 + 2 * s) * F.b_up);     // level 2: nodes 2s, 2s+1
        const uint32_t u3 = bits_at(urow, (48 + s) * F.b_up);         // level 3: node s
        const uint32_t u4 = bits_at(urow, (56 + (s >> 1)) * F.b_up);  // level 4
        const uint32_t u5 = bits_at(urow, (60 + (s >> 2)) * F.b_up);  // level 5
        const uint32_t u6 = bits_at(urow, 62 * F.b_up);               // root
        float S1[4][kG];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint32_t ca, cb;
            if (F.b_leaf == 8) {
                const uint32_t src = m < 2 ? lc0 : lc1;
                ca = (src >> (16 * (m & 1))) & LM;
                cb = (src >> (16 * (m & 1) + 8)) & LM;
            } else {
                ca = (lc0 >> ((2 * m) * F.b_leaf)) & LM;
                cb = (lc0 >> ((2 * m + 1) * F.b_leaf)) & LM;
            }
            const float2 fa = lut_get(lut, LB + ca, lane);
            const float2 fb = lut_get(lut, LB + cb, lane);
            const float2 fu = lut_get(lut, UB + ((u1 >> (m * F.b_up)) & UM), lane);
#pragma unroll
            for (int h = 0; h < kG; ++h) {
                const float L = qr[h][4 * m] * fa.x + qr[h][4 * m + 1] * fa.y;
                const float R = qr[h][4 * m + 2] * fb.x + qr[h][4 * m + 3] * fb.y;
                S1[m][h] = fu.x * L + fu.y * R;
            }
        }
        float S2[2][kG];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const float2 fu = lut_get(lut, UB + ((u2 >> (m * F.b_up)) & UM), lane);
#pragma unroll
            for (int h = 0; h < kG; ++h) S2[m][h] = fu.x * S1[2 * m][h] + fu.y * S1[2 * m + 1][h];
        }
        float S3[kG];
        {
            const float2 fu = lut_get(lut, UB + (u3 & UM), lane);
#pragma unroll
            for (int h = 0; h < kG; ++h) S3[h] = fu.x * S2[0][h] + fu.y * S2[1][h];
        }
        // level 4: lanes s, s^1 hold sibling subtrees; even lane keeps heads 0,1
        const bool odd = s & 1;
        const float r0 = __shfl_xor_sync(full, odd ? S3[0] : S3[2], 1);
        const float r1 = __shfl_xor_sync(full, odd ? S3[1] : S3[3], 1);
        float T0, T1;
        {
            const float2 fu = lut_get(lut, UB + (u4 & UM), lane);
            T0 = fu.x * (odd ? r0 : S3[0]) + fu.y * (odd ? S3[2] : r0);
            T1 = fu.x * (odd ? r1 : S3[1]) + fu.y * (odd ? S3[3] : r1);
        }
        // level 5: lanes s, s^2; bit1 = 0 keeps the first of the pair
        const bool hi1 = (s >> 1) & 1;
        const float r2 = __shfl_xor_sync(full, hi1 ? T0 : T1, 2);
        float U;
        {
            const float2 fu = lut_get(lut, UB + (u5 & UM), lane);
            U = fu.x * (hi1 ? r2 : T0) + fu.y * (hi1 ? T1 : r2);
        }
        // root: lanes s, s^4 (both end with the same value)
        const bool right = (s >> 2) & 1;
        const float r3 = __shfl_xor_sync(full, U, 4);
        float S;
        {
            const float2 fu = lut_get(lut, UB + (u6 & UM), lane);
            S = fu.x * (right ? r3 : U) + fu.y * (right ? U : r3);
        }
        const float rr = __half2float(((const __half*)pg)[t]);
        lg[pass] = t < valid ? rr * S * kLogitScale : -INFINITY;
    }
    // online softmax for this lane's head (lanes k = 0..3 share it)
    float pm = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
    pm = fmaxf(pm, __shfl_xor_sync(full, pm, 8));
    pm = fmaxf(pm, __shfl_xor_sync(full, pm, 16));
    const float m_new = fmaxf(st.m, pm);
    const float alpha = exp2f(st.m - m_new);   // st.m = -inf on the first page -> 0
    st.m = m_new;
    float psum = 0.f;
    const __half* vs = (const __half*)(pg + 2 * kP);
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const float pv = exp2f(lg[pass] - m_new);
        psum += pv;
        if (s < 4) pbuf[(pass * 4 + k) * kG + head] = pv * __half2float(vs[pass * 4 + k]);
    }
    st.l = st.l * alpha + psum;
    if (lane < 4) pbuf[16 * kG + head] = alpha;
    __syncwarp();
    const float4 al = *(const float4*)(pbuf + 16 * kG);
    const float a4[kG] = {al.x, al.y, al.z, al.w};
#pragma unroll
    for (int h = 0; h < kG; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) st.o[h][i] *= a4[h];
    const uint8_t* vrow0 = pg + F.off_v;
    for (int t = 0; t < valid; ++t) {
        const float4 w = *(const float4*)(pbuf + t * kG);
        float v[4];
        if (F.v_bits == 8) {
            const uint32_t x = ld_u32(vrow0 + t * F.v_row + 4 * lane);
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = (float)((int32_t)(x << (24 - 8 * i)) >> 24);
        } else {
            const uint32_t x = *(const uint16_t*)(vrow0 + t * F.v_row + 2 * lane);
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = (float)((int32_t)(x << (28 - 4 * i)) >> 28);
        }
        const float wv[kG] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < kG; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) st.o[h][i] = fmaf(wv[h], v[i], st.o[h][i]);
    }
    __syncwarp();
}

// ------------------------------------------------------------ decode --
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(DecodeParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    float2* lut = (float2*)smem;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const unsigned full = 0xffffffffu;

    // cos/sin tables: leaf grids c*2pi/2^b, upper grids c*(pi/2)/(2^b-1)
    for (int e = tid; e < kLutEntries; e += kThreads) {
        double a;   // angle / pi
        if (e < kLeafBase2) a = (double)e / 128.0;
        else if (e < kLeafBase3) a = (double)(e - kLeafBase2) / 8.0;
        else if (e < kUpBase1) a = (double)(e - kLeafBase3) / 4.0;
        else if (e < kUpBase2) a = (double)(e - kUpBase1) / 510.0;
        else if (e < kUpBase3) a = (double)(e - kUpBase2) / 126.0;
        else a = (double)(e - kUpBase3) / 30.0;
        double sn, cs;
        sincospi(a, &sn, &cs);
        const float2 v = make_float2((float)cs, (float)sn);
#pragma unroll
        for (int r = 0; r < kRep; ++r) lut[e * kRep + r] = v;
    }
    uint8_t* stage = smem + kStageOff + w * kStages * kStageBytes;
    float* pbuf = (float*)(smem + kPbufOff) + w * kPbufFloats;
    const uint32_t bar0 = smem_u32(smem + kBarOff + w * kStages * 8);
    if (lane == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        fence_barrier_init();
    }
    __syncthreads();

    const int32_t P = p.unit_start[p.n_units];
    const int32_t lo = cta_bound(blockIdx.x, P, p.n_cta), hi = cta_bound(blockIdx.x + 1, P, p.n_cta);
    uint32_t phase = 0;   // bit s = parity to wait for on stage s
    bool failed = false;

    float* ms_m = (float*)(smem + kStageOff);   // merge scratch, aliases the ring
    float* ms_l = ms_m + kWarps * kG;
    float* ms_o = ms_l + kWarps * kG;

    for (int32_t x = lo; x < hi;) {
        const int u = find_unit(p.unit_start, p.n_units, x);
        const int32_t us = p.unit_start[u], ue = p.unit_start[u + 1];
        const int32_t seg_end = min(hi, ue);
        const int b = u / p.H_kv, g = u % p.H_kv;
        const int32_t pa = x - us, pe = seg_end - us;   // unit-local page range
        const int64_t first = p.page_offsets[b];
        const int len = p.seq_lens[b];
        const int32_t* ptab = p.page_table + (int64_t)g * p.total_pages + first;

        // this lane's query slice: dims 16s .. 16s+15 of heads 4g .. 4g+3
        float qr[kG][16];
        {
            const int s = lane & 7;
#pragma unroll
            for (int h = 0; h < kG; ++h) {
                const float4* src = (const float4*)(p.q + ((int64_t)b * p.H_q + g * kG + h) * kD + 16 * s);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 v = src[i];
                    qr[h][4 * i] = v.x;
                    qr[h][4 * i + 1] = v.y;
                    qr[h][4 * i + 2] = v.z;
                    qr[h][4 * i + 3] = v.w;
                }
            }
        }
        WarpState st;
        st.m = -INFINITY;
        st.l = 0.f;
#pragma unroll
        for (int h = 0; h < kG; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) st.o[h][i] = 0.f;

        // this warp's pages: pa + w + 16 i.  Entries are read 32 at a time.
        int ebase = 0;
        int32_t ent = 0;
        uint32_t mask = 0;
        auto refill = [&]() {
            const int32_t lp = pa + w + kWarps * (ebase + lane);
            ent = lp < pe ? ptab[lp] : 0;
            int t = entry_tier(ent);
            bool ok = t != 0;
            if (ok && entry_page(ent) >= p.pool_pages[t]) {
                report(p.status, SPHKV_ERR_DATA);
                ok = false;
            }
            mask = __ballot_sync(full, ok);
        };
        auto next = [&](int32_t& lp, int32_t& e) -> bool {
            while (mask == 0) {
                ebase += 32;
                if (pa + w + kWarps * ebase >= pe) return false;
                refill();
            }
            const int j = __ffs(mask) - 1;
            mask &= mask - 1;
            lp = pa + w + kWarps * (ebase + j);
            e = __shfl_sync(full, ent, j);
            return true;
        };
        auto issue = [&](int stg, int32_t e) {
            if (lane == 0) {
                const int t = entry_tier(e);
                const uint32_t bytes = (uint32_t)page_bytes_of(t);
                const uint8_t* src = p.pool[t] + entry_page(e) * (int64_t)bytes;
                fence_proxy_async();
                mbar_expect_tx(bar0 + 8 * stg, bytes);
                bulk_g2s(smem_u32(stage + stg * kStageBytes), src, bytes, bar0 + 8 * stg);
            }
        };
        refill();
        int32_t lp_cur = 0, e_cur = 0, lp_nxt = 0, e_nxt = 0;
        bool have_cur = next(lp_cur, e_cur);
        int cur = 0;
        if (have_cur) issue(0, e_cur);
        while (have_cur) {
            const bool have_nxt = next(lp_nxt, e_nxt);
            if (have_nxt) issue(cur ^ 1, e_nxt);
            const bool ok = mbar_wait(bar0 + 8 * cur, (phase >> cur) & 1);
            phase ^= 1u << cur;
            if (!ok) {
                if (lane == 0) report(p.status, SPHKV_ERR_TIMEOUT);
                failed = true;
                if (have_nxt) {   // drain the copy still in flight, again bounded
                    mbar_wait(bar0 + 8 * (cur ^ 1), (phase >> (cur ^ 1)) & 1);
                    phase ^= 1u << (cur ^ 1);
                }
                break;
            }
            const uint8_t* pg = stage + cur * kStageBytes;
            const int valid = min(kP, len - lp_cur * kP);
            const int t = entry_tier(e_cur);
            if (t == 1) process_page<1>(pg, valid, qr, lut, pbuf, lane, st);
            else if (t == 2) process_page<2>(pg, valid, qr, lut, pbuf, lane, st);
            else process_page<3>(pg, valid, qr, lut, pbuf, lane, st);
            cur ^= 1;
            lp_cur = lp_nxt;
            e_cur = e_nxt;
            have_cur = have_nxt;
        }

        // ---- CTA merge of the 16 warps' (m, l, o) for this segment
        float lt = st.l;   // lanes s and s+4 duplicate: sum over k only
        lt += __shfl_xor_sync(full, lt, 8);
        lt += __shfl_xor_sync(full, lt, 16);
        __syncthreads();   // every warp is done with its ring
        {
            const int s = lane & 7;
            const int head = (s & 1) * 2 + ((s >> 1) & 1);
            if (lane < 4) {
                ms_m[w * kG + head] = st.m;
                ms_l[w * kG + head] = lt;
            }
#pragma unroll
            for (int h = 0; h < kG; ++h)
                *(float4*)(ms_o + (w * kG + h) * kD + 4 * lane) =
                    make_float4(st.o[h][0], st.o[h][1], st.o[h][2], st.o[h][3]);
        }
        __syncthreads();
        {
            const int h = tid >> 7, dim = tid & (kD - 1);
            float M = -INFINITY;
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, ms_m[ww * kG + h]);
            float L = 0.f, O = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int ww = 0; ww < kWarps; ++ww) {
                    const float mw = ms_m[ww * kG + h];
                    if (mw == -INFINITY) continue;
                    const float sc = exp2f(mw - M);
                    L += ms_l[ww * kG + h] * sc;
                    O += ms_o[(ww * kG + h) * kD + dim] * sc;
                }
            }
            if (pa == 0 && seg_end == ue) {   // the whole unit: final result
                const int64_t row = (int64_t)b * p.H_q + g * kG + h;
                p.out[row * kD + dim] = L > 0.f ? O / L : 0.f;
                if (dim == 0) p.lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
            } else {
                float* part = p.partial + ((int64_t)(blockIdx.x + u) * kG + h) * kPartStride;
                part[4 + dim] = O;
                if (dim == 0) {
                    part[0] = M;
                    part[1] = L;
                }
            }
        }
        __syncthreads();   // scratch free before the next segment's copies
        x = seg_end;
        if (failed) break;
    }
}

// --------------------------------------------------------------- merge --
__global__ void __launch_bounds__(kG * kD) merge_kernel(DecodeParams p)
{
    const int u = blockIdx.x;
    const int h = threadIdx.x >> 7, dim = threadIdx.x & (kD - 1);
    const int32_t P = p.unit_start[p.n_units];
    const int32_t us = p.unit_start[u], ue = p.unit_start[u + 1];
    const int b = u / p.H_kv, g = u % p.H_kv;
    const int64_t row = (int64_t)b * p.H_q + g * kG + h;
    if (ue == us) {   // no pages: nothing attended
        p.out[row * kD + dim] = 0.f;
        if (dim == 0) p.lse[row] = -INFINITY;
        return;
    }
    // CTAs whose piece of [0, P) meets [us, ue)
    int c0 = (int)(((int64_t)us * p.n_cta) / P);
    while (c0 > 0 && cta_bound(c0, P, p.n_cta) > us) --c0;
    while (cta_bound(c0 + 1, P, p.n_cta) <= us) ++c0;
    int c1 = c0;
    while (c1 + 1 < p.n_cta && cta_bound(c1 + 1, P, p.n_cta) < ue) ++c1;
    if (c0 == c1) return;   // one CTA finished this unit and wrote it
    // CTAs with an empty piece (possible when P < n_cta * pages) wrote nothing
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c)
        if (cta_bound(c, P, p.n_cta) < cta_bound(c + 1, P, p.n_cta))
            M = fmaxf(M, p.partial[((int64_t)(c + u) * kG + h) * kPartStride]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
        for (int c = c0; c <= c1; ++c) {
            if (cta_bound(c, P, p.n_cta) == cta_bound(c + 1, P, p.n_cta)) continue;
            const float* part = p.partial + ((int64_t)(c + u) * kG + h) * kPartStride;
            if (part[0] == -INFINITY) continue;
            const float sc = exp2f(part[0] - M);
            L += part[1] * sc;
            O += part[4 + dim] * sc;
        }
    }
    p.out[row * kD + dim] = L > 0.f ? O / L : 0.f;
    if (dim == 0) p.lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

int sm_count(int n_sm)
{
    if (n_sm > 0) return n_sm;
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return v;
}

int pick_ctas(int H_kv, int64_t total_pages, int n_sm)
{
    int64_t pmax = (int64_t)H_kv * total_pages;
    int64_t n = (pmax + kMinPagesPerCta - 1) / kMinPagesPerCta;
    if (n < 1) n = 1;
    if (n > n_sm) n = n_sm;
    return (int)n;
}

size_t ws_layout(int B, int H_kv, int n_cta, size_t* part_off)
{
    size_t n_units = (size_t)B * H_kv;
    size_t off = ((n_units + 1) * 4 + 255) / 256 * 256;
    *part_off = off;
    return off + (size_t)(n_cta + n_units) * kG * kPartStride * 4;
}

}  // namespace
}  // namespace sphkv

using namespace sphkv;

extern "C" size_t sphkv_decode_workspace_bytes(int32_t B, int32_t H_q, int32_t H_kv,
                                               int64_t total_pages, int32_t n_sm)
{
    (void)H_q;
    if (B <= 0 || H_kv <= 0 || total_pages < 0) return 0;
    size_t off;
    return ws_layout(B, H_kv, pick_ctas(H_kv, total_pages, sm_count(n_sm)), &off);
}

extern "C" sphkv_status sphkv_decode_attention(const sphkv_cache* c, int32_t H_q, const float* q,
                                               float* out, float* lse, void* workspace,
                                               size_t ws_bytes, int32_t* status_dev, void* stream)
{
    if (!c || !q || !out || !lse || !workspace) {
        sphkv_set_error("sphkv_decode_attention: null argument");
        return SPHKV_ERR_ARG;
    }
    if (c->B <= 0 || c->H_kv <= 0 || !c->page_offsets || !c->seq_lens || !c->page_table ||
        c->total_pages < 0) {
        sphkv_set_error("sphkv_decode_attention: bad cache descriptor");
        return SPHKV_ERR_ARG;
    }
    if (H_q != kG * c->H_kv) {
        sphkv_set_error("sphkv_decode_attention: H_q / H_kv must be %d (got H_q=%d, H_kv=%d)", kG, H_q,
                        c->H_kv);
        return SPHKV_ERR_ARG;
    }
    if (((uintptr_t)q & 15) || ((uintptr_t)workspace & 255)) {
        sphkv_set_error("sphkv_decode_attention: q must be 16-byte and workspace 256-byte aligned");
        return SPHKV_ERR_ARG;
    }
    if ((int64_t)c->H_kv * c->total_pages > 0x7fffffffLL || (int64_t)c->B * c->H_kv > (1 << 24)) {
        sphkv_set_error("sphkv_decode_attention: cache too large for 32-bit page indices");
        return SPHKV_ERR_ARG;
    }
    DecodeParams p{};
    for (int t = 1; t <= 3; ++t) {
        p.pool[t] = c->pool[t - 1];
        p.pool_pages[t] = c->pool[t - 1] ? c->pool_pages[t - 1] : 0;
        if ((uintptr_t)c->pool[t - 1] & 15) {
            sphkv_set_error("sphkv_decode_attention: pool %d is not 16-byte aligned", t);
            return SPHKV_ERR_ARG;
        }
    }
    const int n_sm = sm_count(0);
    p.n_cta = pick_ctas(c->H_kv, c->total_pages, n_sm);
    size_t part_off;
    const size_t need = ws_layout(c->B, c->H_kv, p.n_cta, &part_off);
    if (ws_bytes < need) {
        sphkv_set_error("sphkv_decode_attention: workspace %zu bytes < %zu needed", ws_bytes, need);
        return SPHKV_ERR_ARG;
    }
    p.page_offsets = c->page_offsets;
    p.seq_lens = c->seq_lens;
    p.page_table = c->page_table;
    p.total_pages = c->total_pages;
    p.B = c->B;
    p.H_kv = c->H_kv;
    p.H_q = H_q;
    p.n_units = c->B * c->H_kv;
    p.q = q;
    p.out = out;
    p.lse = lse;
    p.unit_start = (int32_t*)workspace;
    p.partial = (float*)((uint8_t*)workspace + part_off);
    p.status = status_dev;

    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes) != cudaSuccess) {
            sphkv_set_error("sphkv_decode_attention: cannot reserve %d bytes of shared memory", kSmemBytes);
            return SPHKV_ERR_DEVICE;
        }
        attr_dev = dev;
    }
    cudaStream_t s = (cudaStream_t)stream;
    plan_kernel<<<1, 1024, 0, s>>>(p);
    decode_kernel<<<p.n_cta, kThreads, kSmemBytes, s>>>(p);
    merge_kernel<<<p.n_units, kG * kD, 0, s>>>(p);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("sphkv_decode_attention: launch failed: %s", cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}
