// decode.cu -- angle-domain attention (ADA) decode over the paged cache.
//
// Spherical KV (arXiv 2605.18856), Abstract: the logits are computed from the
// angle codes themselves, never from rebuilt dense keys, on a paged,
// block-local decode path whose aim is less HBM traffic.  The logit of query q
// against a stored key is r * S_root / sqrt(d), with S defined bottom-up over
// the recursive-polar tree:
//   leaf j:     S = q[2j] cos(phi_j) + q[2j+1] sin(phi_j)
//   upper node: S = cos(psi) S_left + sin(psi) S_right
// and evaluated here in its unrolled (top-down) form.
// Values are dequantised (int8/int4 code times the token's fp16 scale) inside
// the value FMA; an online softmax keeps (max, sum, out) per query head, and
// long contexts are split across SMs and merged with a log-sum-exp combine.
//
// Launch structure (three kernels on the caller's stream; decode and merge
// are programmatic dependent launches that overlap the previous kernel's
// tail and wait for its results):
//   plan   -- 1 CTA: unit_start[u] = pages before unit u = (b, g), u = b*H_kv+g.
//   decode -- persistent, one 384-thread CTA (12 warps) per SM.  The flattened
//             page range [0, P) is cut into n_cta equal pieces; a CTA walks the
//             units its piece overlaps.  Its warps split each unit's pages into
//             contiguous ranges of equal tier weight; each warp bulk-copies a
//             page (cp.async.bulk, mbarrier completion) into a 2-stage ring in
//             shared memory while it computes the previous one.
//             Logits, top down: 4 tokens per pass, 8 lanes per token; lane
//             (k, s) owns subtree block s (8 leaves, 7 upper nodes) of its
//             token for every head of the unit, gets the three ancestors' codes
//             by shuffle, and forms the leaves' path products once for all
//             heads.  T1 leaves: a (cos, sin) lookup times the path weight,
//             dotted with the lane's query slice in registers.  T2/T3 leaves:
//             one 16-byte lookup in a per-unit table that already holds
//             q[2j] cos(phi) + q[2j+1] sin(phi) for 4 heads.  The tables sit at
//             absolute shared addresses with lane replicas, a code becomes an
//             address with one byte permute (8- and 4-bit codes) or a shift
//             and a masked OR, and the heads are kept in a lane-dependent
//             order so that the 8-lane sum is a select-free reduce-scatter
//             leaving each lane one head; the logits stay in registers into
//             the online softmax.
//             Values: out^T[dims x heads] += V^T[dims x 16 tokens] P^T on the
//             tensor cores (mma.sync m16n8k16, f16 operands, fp32
//             accumulators).  Value codes are exact in f16; the weights
//             p * vscale * sc are split into f16 hi + lo parts, keeping ~22
//             bits (one query: both parts in one MMA, columns 0-3 and 4-7; a
//             pair: two MMAs).
//   merge  -- one CTA per unit; only units whose pages were split over
//             several CTAs do any work.
// decode_kernel<1> serves one query token per sequence (4 query heads per kv
// head); decode_kernel<2> serves a pair of causal query tokens (8 heads), see
// "two query tokens per pass" below.
#include <cstdlib>

#include "common.cuh"

namespace sphkv {
namespace {

constexpr int kG = 4;               // query heads per kv head
constexpr int kStageBytes = Tier<1>::f.page_bytes;  // largest page
constexpr int kMinPagesPerCta = 64;
constexpr int kPartStride = 132;    // floats per (slot, head): m, l, pad, pad, o[128]

// Cos/sin tables, shared by both decode kernels.  T1: one 256-byte row per
// code, [leaf (cos,sin) x 16 lane replicas][upper (cos,sin) x 16 replicas].
// T2, T3: upper grid only, 16 replicas (128 bytes) per code, in 128-byte (T2)
// or 256-byte (T3) rows.  T2 and T3 leaves read the query-folded tables, built
// from T1 leaf rows: the leaf grids nest (T2 code c has the angle of T1 code
// 16c, T3 code c that of T2 code 2c).
//
// Shared-memory layout of decode_kernel<NQ>.  Region offsets are absolute
// shared-window addresses (the dynamic block must start below the first
// region, which the kernel checks), each table placed so that a lookup address
// is the code permuted or OR-ed into the table base and the lane's replica,
// plus an immediate offset: one or two instructions per code, no address add.
template <int NQ>
struct Layout;
// One query token: 12 warps, 8 lanes per token, each lane holding its
// subtree's query slice in registers (168 registers a thread); two-stage page
// rings.  The query-folded T2/T3 leaf table holds, for leaf j = 8s + i and T2
// code c, the 4 heads' q[2j] cos(phi_c) + q[2j+1] sin(phi_c) (times the logit
// scale) at kFold + (i << 12) + (c << 8) + (s << 4), in the head order of the
// lanes that own subtree s: a code byte placed in bits 8..15 of the lane's
// base (s << 4) is the address, leaf i's slab an immediate offset, and the 8
// lanes of a token read 8 distinct bank groups.
template <>
struct Layout<1> {
    static constexpr int kWarps = 12;
    static constexpr int kStages = 2;
    static constexpr int kHeads = kG;
    static constexpr int kPbufFloats = 16 * kG + 2 * kG;   // p*scale per (token, head); alpha per head; valid
    static constexpr uint32_t kUpT2 = 8192;                // 64 rows x 128 B, 8 KB aligned
    static constexpr uint32_t kUpT3 = 16384;               // 16 rows x 256 B (128 B used)
    static constexpr uint32_t kPbuf = 20480;
    static constexpr uint32_t kBar = kPbuf + kWarps * kPbufFloats * 4;
    static constexpr uint32_t kSlice = kBar + kWarps * kStages * 8;
    static constexpr uint32_t kFold = 32768;               // 8 leaf slabs x 16 codes x 256 B
    static constexpr uint32_t kT1 = 65536;                 // 256 rows x 256 B, 64 KB aligned
    static constexpr uint32_t kStage = 131072;
    static constexpr int kSmemBytes = (int)(kStage + kWarps * kStages * kStageBytes);
};
// A pair of query tokens (8 heads): the same absolute plan and lane mapping as
// one query, 12 warps, no query registers.  Lane (k, s) holds, for its subtree
// s, slots i = 0..7 of the unit's 8 heads in the order head(i) = i ^ s (heads
// 0-3: the first query token, 4-7: the second), so that the 8-lane sum leaves
// lane s with head s.  T1 leaves read the query rows kQ (slot pair hp = slots
// 2hp, 2hp+1 of leaf j = 8s + i at kQ + 512 i + 128 hp + 16 s); T2/T3 leaves
// read slots 0-3 from the first folded table and 4-7 from the second (entry of
// T2 code c: kFold + (i << 12) + (c << 8) + (s << 4), the second table's 128
// bytes on).
template <>
struct Layout<2> {
    static constexpr int kWarps = 12;
    static constexpr int kStages = 2;
    static constexpr int kHeads = 2 * kG;
    static constexpr int kPbufFloats = 16 * 2 * kG + 2 * 2 * kG;   // weights; alpha per head
    static constexpr uint32_t kUpT2 = 8192;
    static constexpr uint32_t kUpT3 = 16384;
    static constexpr uint32_t kPbuf = 20480;
    static constexpr uint32_t kBar = kPbuf + kWarps * kPbufFloats * 4;
    static constexpr uint32_t kSlice = kBar + kWarps * kStages * 8;
    static constexpr uint32_t kQ = 27648;                  // 8 leaves x 4 slot pairs x 8 subtrees x 16 B
    static constexpr uint32_t kFold = 32768;               // 8 leaf slabs x 16 codes x 2 tables x 128 B
    static constexpr uint32_t kFold2 = 128;                // second table, from the first
    static constexpr uint32_t kT1 = 65536;
    static constexpr uint32_t kStage = 131072;
    static constexpr int kSmemBytes = (int)(kStage + kWarps * kStages * kStageBytes);
};
template <int NQ>
constexpr bool layout_ok()
{
    using L = Layout<NQ>;
    return L::kStage % 128 == 0 && L::kPbuf % 16 == 0 && L::kBar % 8 == 0 && L::kT1 % 65536 == 0 &&
           L::kUpT2 % 8192 == 0 && L::kUpT3 % 2048 == 0 && L::kSmemBytes <= 227 * 1024 &&
           // CTA merge scratch (aliases the rings): m[W][H], l[W][H], o[W][H][128]
           (2 * L::kWarps * L::kHeads + L::kWarps * L::kHeads * kD) * 4 <=
               L::kWarps * L::kStages * kStageBytes;
}
static_assert(layout_ok<1>() && layout_ok<2>(), "shared-memory layout");
// word after the slice sums: violations seen by the debug build's checks
template <int NQ>
constexpr uint32_t kDbgFlag = Layout<NQ>::kSlice + 4 * Layout<NQ>::kWarps;
static_assert(Layout<1>::kSlice + Layout<1>::kWarps * 4 + 4 <= Layout<1>::kFold && Layout<1>::kFold % 32768 == 0 &&
                  Layout<1>::kFold + 32768 <= Layout<1>::kT1 && Layout<1>::kT1 + 65536 <= Layout<1>::kStage,
              "one-query regions");
static_assert(Layout<2>::kSlice + Layout<2>::kWarps * 4 + 4 <= Layout<2>::kQ && Layout<2>::kQ % 128 == 0 &&
                  Layout<2>::kQ + 4096 <= Layout<2>::kFold && Layout<2>::kFold % 32768 == 0 &&
                  Layout<2>::kFold + 32768 <= Layout<2>::kT1 &&
                  Layout<2>::kT1 + 65536 <= Layout<2>::kStage && Layout<1>::kUpT2 == Layout<2>::kUpT2,
              "pair regions");

constexpr float kLn2 = 0.6931471805599453f;
// log2(e) / sqrt(128): logits are kept in the log2 domain
constexpr float kLogitScale = 0.12751743082459868f;
// The value weights p * vscale are multiplied by a power of two sc before the
// f16 hi/lo split: 2^12 to start with, lowered (with the accumulators
// rescaled) when a page brings a scale with vscale * sc > 2^15, so that a
// weight (p <= 1) never leaves the f16 range.
constexpr float kPScale = 4096.0f;
constexpr float kWeightMax = 32768.0f;

constexpr long kWaitLimit = 1L << 22;

struct DecodeParams {
    const int32_t* page_offsets;
    const int32_t* seq_lens;
    const int32_t* page_table;
    const uint8_t* pool[4];
    int64_t pool_pages[4];
    int64_t total_pages;
    int B, H_kv, H_q, n_units, n_cta;
    // Query tokens per sequence (nq), the first of those this launch handles
    // (q0) and how many it handles (npair, 1 or 2); query token i sees the
    // first seq_len - (nq - 1 - i) tokens.  q, out: [B][nq][H_q][128],
    // lse: [B][nq][H_q].  len_shift = nq - q0 - npair: the launch's page range
    // is that of its last query token.
    int nq, q0, npair, len_shift;
#ifdef SPHKV_TEST_HOOKS
    // Test builds only (environment SPHKV_TEST_SKIP_FIRST_COPY): warp 0 of
    // CTA 0 skips its first page copy and waits with a short limit, so that
    // wait runs out and the call reports SPHKV_ERR_TIMEOUT without any fault;
    // every other warp and CTA runs as in the product build.
    int test_skip_copy;
#endif
    const float* q;
    float* out;
    float* lse;
    int32_t* unit_start;   // [n_units + 1]
    float* partial;        // [n_cta + n_units][heads per unit][kPartStride]
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
template <long Limit = kWaitLimit>
__device__ inline bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (long i = 0; i < Limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (i > 16) __nanosleep(64);
    }
    return false;
}

// ---------------------------------------------------------------- plan --
__global__ void __launch_bounds__(1024) plan_kernel(DecodeParams p)
{
    // let the decode kernel start its prologue now; it waits for this grid's
    // results before it reads them
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
            if (len < 0) report(p.status, SPHKV_ERR_DATA);
            len = len - p.len_shift > 0 ? len - p.len_shift : 0;
            int64_t np = (len + kP - 1) / kP;
            if (np > cap) {
                report(p.status, SPHKV_ERR_DATA);
                np = cap;
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

// Work of a page by tier, for splitting a CTA's pages among its warps, set
// from measurements of each kernel: one query, T1 5 : T2/T3 6 (a T1 page
// carries 1.8x the bytes but its leaves are cheaper than folded ones); a
// pair, T1 5 : T2/T3 3 (its T1 leaves read query rows from shared memory).
// A dropped page weighs 0 and is skipped.
template <int NQ>
__device__ __forceinline__ uint32_t page_weight(int32_t e)
{
    const int t = entry_tier(e);
    if (NQ == 1) return t == 0 ? 0u : t == 1 ? 5u : 6u;
    return t == 0 ? 0u : t == 1 ? 5u : 3u;
}

// ------------------------------------------------------------- page work --
struct WarpState {
    float m;             // running max (log2 domain) of this lane's head
    float l;             // running sum of this lane's tokens
    float sc;            // power of two: value weights are p * vscale * sc
    float acc[8][4];     // MMA accumulators (in units of 1 / sc): tile m = dims 16m..16m+15
};

// Largest power of two <= x (x positive and normal).
__device__ __forceinline__ float pow2_floor(float x)
{
    return __int_as_float(__float_as_int(x) & 0x7f800000);
}

template <int T>
__device__ __forceinline__ uint32_t shift_mask(uint32_t x, int sh, uint32_t mask)
{
    return (sh >= 0 ? x << sh : x >> -sh) & mask;
}

// 2^x on the special-function unit (max relative error about 2^-22); -inf -> 0.
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two halves packed as f16x2: `lo` in the low half.
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi)
{
    const __half2 h = __floats2half2_rn(lo, hi);
    return *(const uint32_t*)&h;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory loads by 32-bit shared address (the lookups below build full
// addresses; these keep the compiler from adding a base to each).
template <int Off = 0>
__device__ __forceinline__ float lds32(uint32_t a)
{
    float v;
    asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(Off));
    return v;
}
template <int Off = 0>
__device__ __forceinline__ float2 lds64(uint32_t a)
{
    float2 v;
    asm("ld.shared.v2.f32 {%0, %1}, [%2+%3];" : "=f"(v.x), "=f"(v.y) : "r"(a), "n"(Off));
    return v;
}
template <int Off = 0>
__device__ __forceinline__ float4 lds128(uint32_t a)
{
    float4 v;
    asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a), "n"(Off));
    return v;
}

// Shared addresses (before the immediate offset of the table) of the 8 leaf
// and 8 upper lookups of one subtree block.  rep1 = kT1 | leaf replica; repU
// = the upper table (kT1 for T1, kUpT2 for T2, none for T3) | upper replica;
// fb = the lane's folded-table column (s << 4).  T1: row addresses, the code
// byte permuted into bits 8..15 (the upper half of a row is 128 bytes on).
// T2 leaves and T3 uppers: 4-bit codes, masked into bytes and permuted into
// bits 8..15 the same way (T3 upper rows are 256 bytes apart).  T3 leaves:
// code c is T2 code 2c, shifted to bit 9.  T2 uppers: 6-bit codes of a 48-bit
// field, one 128-byte row each.
template <int T>
__device__ __forceinline__ void block_addrs(const uint8_t* codes, int blk, uint32_t rep1, uint32_t repU,
                                            uint32_t fb, uint32_t (&lo)[8], uint32_t (&uo)[8])
{
    if (T == 1) {   // byte codes: one permute places the code in bits 8..15 under the base
        const uint4 w = *(const uint4*)(codes + blk * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            lo[j] = __byte_perm(w.x, rep1, 0x7604 | (j << 4));
            lo[4 + j] = __byte_perm(w.y, rep1, 0x7604 | (j << 4));
            uo[j] = __byte_perm(w.z, repU, 0x7604 | (j << 4));
            uo[4 + j] = __byte_perm(w.w, repU, 0x7604 | (j << 4));
        }
    } else if (T == 2) {   // leaf nibbles; upper code j = bits 6j..6j+5 of the 48-bit field h:w.y
        const uint2 w = *(const uint2*)(codes + blk * 8);
        const uint32_t h = *(const uint16_t*)(codes + kP * 64 + blk * 2);
        const uint32_t even = w.x & 0x0F0F0F0Fu, odd = (w.x >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            lo[2 * k] = __byte_perm(even, fb, 0x7604 | (k << 4));
            lo[2 * k + 1] = __byte_perm(odd, fb, 0x7604 | (k << 4));
        }
        constexpr uint32_t kUpMask = 63u << 7;
        uo[0] = ((w.y << 7) & kUpMask) | repU;
        uo[1] = ((w.y << 1) & kUpMask) | repU;
        uo[2] = ((w.y >> 5) & kUpMask) | repU;
        uo[3] = ((w.y >> 11) & kUpMask) | repU;
        uo[4] = ((w.y >> 17) & kUpMask) | repU;
        uo[5] = (__funnelshift_r(w.y, h, 23) & kUpMask) | repU;
        uo[6] = ((h << 3) & kUpMask) | repU;
        uo[7] = ((h >> 3) & kUpMask) | repU;
    } else {   // upper nibbles; leaf code j = bits 3j..3j+2 of the 24-bit field l8:l16
        const uint32_t u = *(const uint32_t*)(codes + blk * 4);
        const uint32_t lf = *(const uint16_t*)(codes + kP * 32 + blk * 2) | ((uint32_t)codes[kP * 48 + blk] << 16);
        const uint32_t even = u & 0x0F0F0F0Fu, odd = (u >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uo[2 * k] = __byte_perm(even, repU, 0x7604 | (k << 4));
            uo[2 * k + 1] = __byte_perm(odd, repU, 0x7604 | (k << 4));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) lo[j] = shift_mask<T>(lf, 9 - 3 * j, 7u << 9) | fb;
    }
}

#ifdef SPHKV_DEBUG
// Debug builds (-DSPHKV_DEBUG) check every table address a subtree block
// computes against the table it indexes: the load's address (register plus
// immediate) must lie inside the table and be aligned to the load's width.  A
// bad address sets the CTA's flag word (reported as SPHKV_ERR_DEVICE at the
// end of the segment) and is replaced by one inside the table, so the checked
// build never reads outside its tables either.
template <int NQ>
__device__ __forceinline__ void dbg_fix(uint32_t& a, uint32_t imm, uint32_t base, uint32_t size, uint32_t align)
{
    const uint32_t x = a + imm;
    if (x < base || x + align > base + size || (x & (align - 1))) {
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(kDbgFlag<NQ>), "r"(1u) : "memory");
        a = base - imm;
    }
}

// lo: leaf lookups (T1 rows, or the folded table(s) with leaf j's slab at
// 4096 j and, for a pair, the second table 128 bytes on); uo: upper lookups.
template <int NQ, int T>
__device__ __forceinline__ void dbg_check_block(uint32_t (&lo)[8], uint32_t (&uo)[8])
{
    using L = Layout<NQ>;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (T == 1) {
            dbg_fix<NQ>(lo[j], 0, L::kT1, 65536, 8);
            if (lo[j] & 128u) {   // a leaf address must stay in the leaf half of its row
                asm volatile("st.shared.u32 [%0], %1;" ::"r"(kDbgFlag<NQ>), "r"(1u) : "memory");
                lo[j] &= ~128u;
            }
            dbg_fix<NQ>(uo[j], 128, L::kT1, 65536, 8);
        } else {
            dbg_fix<NQ>(lo[j], L::kFold + 4096 * j, L::kFold + 4096 * j, 4096, 16);
            if (NQ == 2) dbg_fix<NQ>(lo[j], L::kFold + 4096 * j + 128, L::kFold + 4096 * j, 4096, 16);
            if (T == 2) dbg_fix<NQ>(uo[j], 0, L::kUpT2, 8192, 8);
            else dbg_fix<NQ>(uo[j], L::kUpT3, L::kUpT3, 4096, 8);
        }
    }
}
#endif

// Logits of the 16 tokens of one page of tier T staged at `pg`, in the log2
// domain: lane (k4, s) ends with lg[pass] = the logit of token 4 pass + k4 for
// head 2 b2 + b1 (s = 4 b2 + 2 b1 + b0).  Eight lanes per token, four tokens per
// pass: lane (k4, s) = (lane >> 3, lane & 7) evaluates subtree s (leaves
// 8s..8s+7, the level-3 node s and the six upper nodes below it) of token
// 4 pass + k4 for all 4 query heads, top down: the tree's value r S_root is
// the sum over leaves of (product of the factors on the leaf's path: cos(psi)
// into a left child, sin(psi) into a right one) times the leaf term
// q[2j] cos(phi_j) + q[2j+1] sin(phi_j).  The three ancestors above level 3
// (level-4 node s/2, level-5 node s/4, the root) are the top codes held in
// slot 7 of blocks s/2, 4 + s/4 and 6, fetched by shuffles; each lane reads
// only the factor on its own side.  The path products do not depend on the
// head.  T1 leaves: (cos, sin) from the table times the path weight, then one
// packed multiply-add per head with the lane's query slice (q[16s..16s+15] of
// the 4 heads, logit scale included) in registers.  T2/T3 leaves: one 16-byte
// lookup of the unit's query-folded table, two packed multiply-adds
// (even and odd leaves in separate chains, added at the end).  Both
// keep the heads in the lane's slot order (slot i holds head ((i >> 1) ^ b2)
// * 2 + ((i & 1) ^ b1) for s = 4 b2 + 2 b1 + b0), which makes the 8-lane sum
// a select-free reduce-scatter that leaves head 2 b2 + b1 in lanes b0 = 0, 1.
template <int T>
__device__ __forceinline__ void page_logits(const uint8_t* pg, int lane, const float2 (&qp)[kG][8], float (&lg)[4])
{
    using L = Layout<1>;
    const unsigned full = 0xffffffffu;
    const int s = lane & 7;
    const uint32_t rep = (uint32_t)(lane & 15) << 3;
    const uint32_t rep1 = L::kT1 | rep;
    const uint32_t repU = (T == 1 ? L::kT1 : T == 2 ? L::kUpT2 : 0u) | rep;
    const uint32_t fb = (uint32_t)s << 4;
    // immediate offset of the upper (cos, sin): inside a T1 row, or the T3 table
    constexpr int kUp = T == 1 ? 128 : T == 2 ? 0 : (int)L::kUpT3;
    // own side at levels 4, 5 and the root (the upper half of a T1 row)
    const uint32_t side4 = (uint32_t)(s & 1) << 2, side5 = (uint32_t)((s >> 1) & 1) << 2,
                   side6 = (uint32_t)(s >> 2) << 2;
    const int grp = lane & ~7;
    const uint8_t* codes = pg + Tier<1>::f.off_codes;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int t = pass * 4 + (lane >> 3);
        uint32_t lo[8], uo[8];
        block_addrs<T>(codes, pass * 32 + lane, rep1, repU, fb, lo, uo);
#ifdef SPHKV_DEBUG
        dbg_check_block<1, T>(lo, uo);
#endif
        // ancestors: top node s/2 (level 4), 4 + s/4 (level 5), 6 (root)
        const uint32_t o4 = __shfl_sync(full, uo[7], grp + (s >> 1));
        const uint32_t o5 = __shfl_sync(full, uo[7], grp + 4 + (s >> 2));
        const uint32_t o6 = __shfl_sync(full, uo[7], grp + 6);
        // radius bits: the sign bit is the token's drop flag, the rest the radius
        // (a flagged token's logit is replaced by -inf, so its sign is left in)
        const uint32_t rb = ((const uint16_t*)pg)[t];
        float v = __half2float(__ushort_as_half((unsigned short)rb));
        v *= lds32<kUp>(o6 | side6);
        v *= lds32<kUp>(o5 | side5);
        v *= lds32<kUp>(o4 | side4);
        float w2[2], w1[4], wl[8];
        {
            const float2 f = lds64<kUp>(uo[6]);
            w2[0] = v * f.x;
            w2[1] = v * f.y;
        }
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const float2 f = lds64<kUp>(uo[4 + n]);
            w1[2 * n] = w2[n] * f.x;
            w1[2 * n + 1] = w2[n] * f.y;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 f = lds64<kUp>(uo[m]);
            wl[2 * m] = w1[m] * f.x;
            wl[2 * m + 1] = w1[m] * f.y;
        }
        float a[kG];
        if (T == 1) {
            float2 acc[kG];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 f = lds64(lo[j]);
                const float2 kk = make_float2(wl[j] * f.x, wl[j] * f.y);
#pragma unroll
                for (int i = 0; i < kG; ++i)
                    acc[i] = j == 0 ? __fmul2_rn(qp[i][j], kk) : __ffma2_rn(qp[i][j], kk, acc[i]);
            }
#pragma unroll
            for (int i = 0; i < kG; ++i) a[i] = acc[i].x + acc[i].y;
        } else {
            float2 acc01[2], acc23[2];   // even and odd leaves: two chains per head pair
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float4 F;
                switch (j) {   // leaf j's slab is 4 KB on
                case 0: F = lds128<L::kFold>(lo[j]); break;
                case 1: F = lds128<L::kFold + 4096>(lo[j]); break;
                case 2: F = lds128<L::kFold + 8192>(lo[j]); break;
                case 3: F = lds128<L::kFold + 12288>(lo[j]); break;
                case 4: F = lds128<L::kFold + 16384>(lo[j]); break;
                case 5: F = lds128<L::kFold + 20480>(lo[j]); break;
                case 6: F = lds128<L::kFold + 24576>(lo[j]); break;
                default: F = lds128<L::kFold + 28672>(lo[j]); break;
                }
                const float2 ww = make_float2(wl[j], wl[j]);
                const int e = j & 1;
                acc01[e] = j < 2 ? __fmul2_rn(ww, make_float2(F.x, F.y)) : __ffma2_rn(ww, make_float2(F.x, F.y), acc01[e]);
                acc23[e] = j < 2 ? __fmul2_rn(ww, make_float2(F.z, F.w)) : __ffma2_rn(ww, make_float2(F.z, F.w), acc23[e]);
            }
            const float2 s01 = __fadd2_rn(acc01[0], acc01[1]), s23 = __fadd2_rn(acc23[0], acc23[1]);
            a[0] = s01.x;
            a[1] = s01.y;
            a[2] = s23.x;
            a[3] = s23.y;
        }
        const float r0 = a[0] + __shfl_xor_sync(full, a[2], 4);
        const float r1 = a[1] + __shfl_xor_sync(full, a[3], 4);
        const float x = r0 + __shfl_xor_sync(full, r1, 2);
        // rotate: after the last pass lg[i] holds pass i
        lg[0] = lg[1];
        lg[1] = lg[2];
        lg[2] = lg[3];
        const float y = x + __shfl_xor_sync(full, x, 1);
        lg[3] = (rb & 0x8000u) ? -INFINITY : y;
    }
}

// Values on the tensor cores for one staged page: out^T[dims x heads] +=
// V^T[dims x 16 tokens] P^T[16 x GQ heads], with the weights P already in
// pbuf[t * GQ + head] and the per-head rescale factor at pbuf[16 GQ + head].
// The weights are split into f16 hi + lo parts.  Four heads (one query token):
// column n holds the hi parts of head n for n < 4 and the lo parts of head
// n - 4 for n >= 4, so one MMA per tile takes both, and the two halves of the
// accumulator are summed at the end (lanes c and c ^ 2).  Eight heads: the hi
// and lo parts go through two MMAs into the same accumulator.
// Thread (g, c): B column g, rows = tokens 2c, 2c+1 (b0) and 2c+8, 2c+9 (b1);
// accumulator columns = heads 2c, 2c+1 (mod GQ).
template <int GQ>
__device__ __forceinline__ void page_values(const uint8_t* pg, int tier, const float* pbuf, int lane, float alpha_acc,
                                            WarpState& st)
{
    const unsigned full = 0xffffffffu;
    const int g = lane >> 2, c = lane & 3;
    if (__any_sync(full, alpha_acc != 1.f)) {   // a running max or sc moved: rescale (rare after the first pages)
        const float2 al = *(const float2*)(pbuf + 16 * GQ + (2 * c) % GQ);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            st.acc[m][0] *= al.x;
            st.acc[m][1] *= al.y;
            st.acc[m][2] *= al.x;
            st.acc[m][3] *= al.y;
        }
    }
    constexpr bool kSplit = GQ == kG;   // hi and lo parts side by side in one tile
    uint32_t bh0 = 0, bh1 = 0, bl0 = 0, bl1 = 0;
    if (kSplit || g < GQ) {
        const int hg = g % GQ;
        const float p0 = pbuf[(2 * c) * GQ + hg], p1 = pbuf[(2 * c + 1) * GQ + hg];
        const float p2 = pbuf[(2 * c + 8) * GQ + hg], p3 = pbuf[(2 * c + 9) * GQ + hg];
        const __half2 h01 = __floats2half2_rn(p0, p1), h23 = __floats2half2_rn(p2, p3);
        bh0 = *(const uint32_t*)&h01;
        bh1 = *(const uint32_t*)&h23;
        bl0 = pack_h2(p0 - __low2float(h01), p1 - __high2float(h01));
        bl1 = pack_h2(p2 - __low2float(h23), p3 - __high2float(h23));
        if (kSplit && g >= GQ) {
            bh0 = bl0;
            bh1 = bl1;
        }
    }
    // rows of tokens 2c, 2c+1, 2c+8, 2c+9 at positions 16g..16g+15; tokens past
    // `valid` carry weight 0 (their rows may hold anything finite)
    if (tier == 1) {
        constexpr TierFmt F = Tier<1>::f;
        const uint8_t* vrow = pg + F.off_v;
        const __half2 bias = __floats2half2_rn(-1152.f, -1152.f);
        // chunk g of row r sits at chunk g ^ (r & 6); r & 6 = 2c for all four rows
        const int ch = 16 * (g ^ (2 * c));
        const uint4 X = *(const uint4*)(vrow + (2 * c) * F.v_row + ch);
        const uint4 Y = *(const uint4*)(vrow + (2 * c + 1) * F.v_row + ch);
        const uint4 Z = *(const uint4*)(vrow + (2 * c + 8) * F.v_row + ch);
        const uint4 W = *(const uint4*)(vrow + (2 * c + 9) * F.v_row + ch);
        const uint32_t xs[4] = {X.x ^ 0x80808080u, X.y ^ 0x80808080u, X.z ^ 0x80808080u, X.w ^ 0x80808080u};
        const uint32_t ys[4] = {Y.x ^ 0x80808080u, Y.y ^ 0x80808080u, Y.z ^ 0x80808080u, Y.w ^ 0x80808080u};
        const uint32_t zs[4] = {Z.x ^ 0x80808080u, Z.y ^ 0x80808080u, Z.z ^ 0x80808080u, Z.w ^ 0x80808080u};
        const uint32_t ws[4] = {W.x ^ 0x80808080u, W.y ^ 0x80808080u, W.z ^ 0x80808080u, W.w ^ 0x80808080u};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int wi = m >> 1, b = 2 * (m & 1);   // byte b (h = 0) and b + 1 (h = 1) of word wi
            // interleave the two tokens' bytes b, b+1, then put 0x64 above each
            // byte: f16 1024 + u with u = code + 128
            const uint32_t sel = (uint32_t)(b | ((4 + b) << 4) | ((b + 1) << 8) | ((5 + b) << 12));
            const uint32_t xy = __byte_perm(xs[wi], ys[wi], sel), zw = __byte_perm(zs[wi], ws[wi], sel);
            uint32_t a[4];
            a[0] = __byte_perm(xy, 0x64646464u, 0x5140);
            a[1] = __byte_perm(xy, 0x64646464u, 0x5342);
            a[2] = __byte_perm(zw, 0x64646464u, 0x5140);
            a[3] = __byte_perm(zw, 0x64646464u, 0x5342);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __half2 hv = __hadd2(*(const __half2*)&a[i], bias);
                a[i] = *(const uint32_t*)&hv;
            }
            mma_16816(st.acc[m], a, bh0, bh1);
            if (!kSplit) mma_16816(st.acc[m], a, bl0, bl1);
        }
    } else {   // T2 and T3 share the int4 row format
        const uint8_t* vrow = pg + (tier == 2 ? Tier<2>::f.off_v : Tier<3>::f.off_v);
        const __half2 bias = __floats2half2_rn(-1032.f, -1032.f);
        const __half2 inv16 = __floats2half2_rn(0.0625f, 0.0625f), bias16 = __floats2half2_rn(-72.f, -72.f);
        // tokens 2i, 2i+1 share a 128-byte block; chunk g ^ (2i & 6) holds 8
        // bytes of each.  Pairs c and c + 4 both give 2i & 6 = 2c.
        const int ch = 16 * (g ^ (2 * c));
        const uint4 XY = *(const uint4*)(vrow + c * 128 + ch);
        const uint4 ZW = *(const uint4*)(vrow + (c + 4) * 128 + ch);
        const uint32_t xs[2] = {XY.x, XY.y}, ys[2] = {XY.z, XY.w};
        const uint32_t zs[2] = {ZW.x, ZW.y}, ws[2] = {ZW.z, ZW.w};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int wi = m >> 2, b = m & 3;   // byte m: low nibble h = 0, high nibble h = 1
            const uint32_t sel = (uint32_t)(b | ((4 + b) << 8));
            const uint32_t xy = __byte_perm(xs[wi], ys[wi], sel);
            const uint32_t zw = __byte_perm(zs[wi], ws[wi], sel);
            // low nibble: f16 1024 + u; high nibble in place: f16 1024 + 16 u,
            // scaled by 1/16 in the bias step (all exact in f16).  u = v + 8
            // (offset binary) is the nibble's top bit flipped, folded with the
            // mask and the exponent bits into one (x & mask) ^ pattern.
            uint32_t a[4];
            a[0] = (xy & 0x000F000Fu) ^ 0x64086408u;
            a[1] = (xy & 0x00F000F0u) ^ 0x64806480u;
            a[2] = (zw & 0x000F000Fu) ^ 0x64086408u;
            a[3] = (zw & 0x00F000F0u) ^ 0x64806480u;
#pragma unroll
            for (int i = 0; i < 4; i += 2) {
                const __half2 lo = __hadd2(*(const __half2*)&a[i], bias);
                const __half2 hi = __hfma2(*(const __half2*)&a[i + 1], inv16, bias16);
                a[i] = *(const uint32_t*)&lo;
                a[i + 1] = *(const uint32_t*)&hi;
            }
            mma_16816(st.acc[m], a, bh0, bh1);
            if (!kSplit) mma_16816(st.acc[m], a, bl0, bl1);
        }
    }
}

// One page of tier `tier` already staged in shared memory at `pg`.  The logits
// are tier-specialised; the softmax and the value MMAs are one copy of code
// for all tiers apart from the value conversion.
__device__ __forceinline__ void process_page(const uint8_t* pg, int tier, int valid, float* pbuf, int lane,
                                             const float2 (&qp)[kG][8], WarpState& st)
{
    const unsigned full = 0xffffffffu;
    const int k = lane >> 3, s = lane & 7;
    const int head = (s >> 2) * 2 + ((s >> 1) & 1);   // lanes b0 = 0, 1 hold the same head
    float lg[4];   // tokens 4 pass + k of this lane's head
    if (tier == 1) page_logits<1>(pg, lane, qp, lg);
    else if (tier == 2) page_logits<2>(pg, lane, qp, lg);
    else page_logits<3>(pg, lane, qp, lg);
#pragma unroll
    for (int pass = 0; pass < 4; ++pass)   // slots past `valid` (last page) get -inf
        if (pass * 4 + k >= valid) lg[pass] = -INFINITY;
    // online softmax for this lane's head (lanes k = 0..3 share it)
    float pm = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
    pm = fmaxf(pm, __shfl_xor_sync(full, pm, 8));
    pm = fmaxf(pm, __shfl_xor_sync(full, pm, 16));
    const float m_new = fmaxf(st.m, pm);
    // no kept token yet (every token so far dropped): any finite shift works
    const float m_ref = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = fast_exp2(st.m - m_ref);   // st.m = -inf on the first page -> 0
    st.m = m_new;
    const __half* vs = (const __half*)(pg + 2 * kP);
    float wv[4];   // vscale * sc of this lane's tokens
    bool big = false;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int t = pass * 4 + k;   // slots past `valid` may hold stale scales: weight exactly 0
        wv[pass] = t < valid ? __half2float(vs[t]) * st.sc : 0.f;
        big |= wv[pass] > kWeightMax;
    }
    float alpha_acc = alpha;
    if (__any_sync(full, big)) {   // rare: lower sc so every weight fits f16
        float vm = fmaxf(fmaxf(wv[0], wv[1]), fmaxf(wv[2], wv[3]));
        vm = fmaxf(vm, __shfl_xor_sync(full, vm, 8));
        vm = fmaxf(vm, __shfl_xor_sync(full, vm, 16));
        const float ratio = pow2_floor(kWeightMax / vm);   // exact: both powers of two scale exactly
        st.sc *= ratio;
        alpha_acc *= ratio;
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) wv[pass] *= ratio;
    }
    float psum = 0.f;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const float pv = fast_exp2(lg[pass] - m_ref);   // -inf (dropped, past the end) -> 0
        psum += pv;
        const int t = pass * 4 + k;
        if (!(s & 1)) pbuf[t * kG + head] = pv * wv[pass];
    }
    st.l = st.l * alpha + psum;
    if (lane < 8 && !(s & 1)) pbuf[16 * kG + head] = alpha_acc;
    __syncwarp();

    page_values<kG>(pg, tier, pbuf, lane, alpha_acc, st);
    __syncwarp();
}

// ---------------------------------------------- two query tokens per pass --
// Several decode query tokens per sequence (speculative or chunked decode):
// a launch takes a pair of them, i.e. 8 query heads per kv head, so one page
// stream, one code unpack and one set of path products serve both tokens,
// and the tensor-core tile's 8 columns are all used.
constexpr int kGQ2 = 2 * kG;                          // heads per unit

// Logits of the 16 tokens of one page for the 8 heads of a query pair, in
// the log2 domain: lane (k4, s) ends with lg[pass] = the logit of token
// 4 pass + k4 for head s.  The lane mapping, the code unpack and the path
// products are page_logits'; the leaf terms go to 8 slots (slot i: head i ^ s).
// T1: (w cos phi, w sin phi) times the 8 slots' query pairs, four 16-byte
// rows in shared memory (the four token groups of the warp read the same
// rows), summed slot pair by slot pair: slot i of lane s' goes straight to
// lane s' ^ i.  T2/T3: one 16-byte lookup in each of the two folded tables,
// then a select-free reduce-scatter (xor 4, 2, 1).  Either way lane s ends
// with head s.
template <int T>
__device__ __forceinline__ void page_logits_pair(const uint8_t* pg, int lane, float (&lg)[4])
{
    using L = Layout<2>;
    const unsigned full = 0xffffffffu;
    const int s = lane & 7;
    const uint32_t rep = (uint32_t)(lane & 15) << 3;
    const uint32_t rep1 = L::kT1 | rep;
    const uint32_t repU = (T == 1 ? L::kT1 : T == 2 ? L::kUpT2 : 0u) | rep;
    const uint32_t fb = (uint32_t)s << 4;
    const uint32_t qb = L::kQ | ((uint32_t)s << 4);
    constexpr int kUp = T == 1 ? 128 : T == 2 ? 0 : (int)L::kUpT3;
    const uint32_t side4 = (uint32_t)(s & 1) << 2, side5 = (uint32_t)((s >> 1) & 1) << 2,
                   side6 = (uint32_t)(s >> 2) << 2;
    const int grp = lane & ~7;
    const uint8_t* codes = pg + Tier<1>::f.off_codes;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int t = pass * 4 + (lane >> 3);
        uint32_t lo[8], uo[8];
        block_addrs<T>(codes, pass * 32 + lane, rep1, repU, fb, lo, uo);
#ifdef SPHKV_DEBUG
        dbg_check_block<2, T>(lo, uo);
#endif
        const uint32_t o4 = __shfl_sync(full, uo[7], grp + (s >> 1));
        const uint32_t o5 = __shfl_sync(full, uo[7], grp + 4 + (s >> 2));
        const uint32_t o6 = __shfl_sync(full, uo[7], grp + 6);
        const uint32_t rb = ((const uint16_t*)pg)[t];   // the sign bit is the token's drop flag
        float v = __half2float(__ushort_as_half((unsigned short)rb));
        v *= lds32<kUp>(o6 | side6);
        v *= lds32<kUp>(o5 | side5);
        v *= lds32<kUp>(o4 | side4);
        float w2[2], w1[4], wl[8];
        {
            const float2 f = lds64<kUp>(uo[6]);
            w2[0] = v * f.x;
            w2[1] = v * f.y;
        }
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const float2 f = lds64<kUp>(uo[4 + n]);
            w1[2 * n] = w2[n] * f.x;
            w1[2 * n + 1] = w2[n] * f.y;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 f = lds64<kUp>(uo[m]);
            wl[2 * m] = w1[m] * f.x;
            wl[2 * m + 1] = w1[m] * f.y;
        }
        float z;   // head s of this lane's token, summed over the token's 8 lanes
        if (T == 1) {
            float2 kk[8];   // (w cos phi, w sin phi) of the block's leaves
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 f = lds64(lo[j]);
                kk[j] = make_float2(wl[j] * f.x, wl[j] * f.y);
            }
            // slot i of lane s' belongs to lane s' ^ i: each slot pair's sums go
            // straight to their lanes (a rolled loop keeps the row loads of one
            // slot pair in flight at a time)
            z = 0.f;
#pragma unroll 1
            for (int hp = 0; hp < 4; ++hp) {   // (q[2j'], q[2j'+1]) of slots 2 hp, 2 hp + 1
                const uint32_t qr = qb + 128u * hp;
                float2 ua, uc;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float4 Q;
                    switch (j) {
                    case 0: Q = lds128<0>(qr); break;
                    case 1: Q = lds128<512>(qr); break;
                    case 2: Q = lds128<1024>(qr); break;
                    case 3: Q = lds128<1536>(qr); break;
                    case 4: Q = lds128<2048>(qr); break;
                    case 5: Q = lds128<2560>(qr); break;
                    case 6: Q = lds128<3072>(qr); break;
                    default: Q = lds128<3584>(qr); break;
                    }
                    const float2 qa = make_float2(Q.x, Q.y), qc = make_float2(Q.z, Q.w);
                    ua = j == 0 ? __fmul2_rn(qa, kk[j]) : __ffma2_rn(qa, kk[j], ua);
                    uc = j == 0 ? __fmul2_rn(qc, kk[j]) : __ffma2_rn(qc, kk[j], uc);
                }
                z += __shfl_xor_sync(full, ua.x + ua.y, 2 * hp);
                z += __shfl_xor_sync(full, uc.x + uc.y, 2 * hp + 1);
            }
        } else {
            float2 acc[4];   // slot pairs (0,1), (2,3), (4,5), (6,7)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float4 F, G;
                switch (j) {   // leaf j's slab is 4 KB on; the second table 128 bytes on
                case 0: F = lds128<L::kFold>(lo[j]); G = lds128<L::kFold + L::kFold2>(lo[j]); break;
                case 1: F = lds128<L::kFold + 4096>(lo[j]); G = lds128<L::kFold + 4096 + L::kFold2>(lo[j]); break;
                case 2: F = lds128<L::kFold + 8192>(lo[j]); G = lds128<L::kFold + 8192 + L::kFold2>(lo[j]); break;
                case 3: F = lds128<L::kFold + 12288>(lo[j]); G = lds128<L::kFold + 12288 + L::kFold2>(lo[j]); break;
                case 4: F = lds128<L::kFold + 16384>(lo[j]); G = lds128<L::kFold + 16384 + L::kFold2>(lo[j]); break;
                case 5: F = lds128<L::kFold + 20480>(lo[j]); G = lds128<L::kFold + 20480 + L::kFold2>(lo[j]); break;
                case 6: F = lds128<L::kFold + 24576>(lo[j]); G = lds128<L::kFold + 24576 + L::kFold2>(lo[j]); break;
                default: F = lds128<L::kFold + 28672>(lo[j]); G = lds128<L::kFold + 28672 + L::kFold2>(lo[j]); break;
                }
                const float2 ww = make_float2(wl[j], wl[j]);
                acc[0] = j == 0 ? __fmul2_rn(ww, make_float2(F.x, F.y)) : __ffma2_rn(ww, make_float2(F.x, F.y), acc[0]);
                acc[1] = j == 0 ? __fmul2_rn(ww, make_float2(F.z, F.w)) : __ffma2_rn(ww, make_float2(F.z, F.w), acc[1]);
                acc[2] = j == 0 ? __fmul2_rn(ww, make_float2(G.x, G.y)) : __ffma2_rn(ww, make_float2(G.x, G.y), acc[2]);
                acc[3] = j == 0 ? __fmul2_rn(ww, make_float2(G.z, G.w)) : __ffma2_rn(ww, make_float2(G.z, G.w), acc[3]);
            }
            // reduce-scatter: slot i pairs with slot i + 4 (xor 4), i + 2 (xor 2), i + 1
            const float x0 = acc[0].x + __shfl_xor_sync(full, acc[2].x, 4);
            const float x1 = acc[0].y + __shfl_xor_sync(full, acc[2].y, 4);
            const float x2 = acc[1].x + __shfl_xor_sync(full, acc[3].x, 4);
            const float x3 = acc[1].y + __shfl_xor_sync(full, acc[3].y, 4);
            const float y0 = x0 + __shfl_xor_sync(full, x2, 2), y1 = x1 + __shfl_xor_sync(full, x3, 2);
            z = y0 + __shfl_xor_sync(full, y1, 1);
        }
        lg[0] = lg[1];
        lg[1] = lg[2];
        lg[2] = lg[3];
        lg[3] = (rb & 0x8000u) ? -INFINITY : z;
    }
}

// One staged page for a query pair.  valid0 / valid1: tokens of the page the
// pair's first / second query sees (the second sees one more token; 0 when
// the launch has one query).  A head that has seen no token yet keeps an
// empty state (max -inf, sum 0).
__device__ __forceinline__ void process_page_pair(const uint8_t* pg, int tier, int valid0, int valid1, float* pbuf,
                                                  int lane, WarpState& st)
{
    const unsigned full = 0xffffffffu;
    const int k = lane >> 3, s = lane & 7;   // head s, tokens 4 pass + k
    float lg[4];
    if (tier == 1) page_logits_pair<1>(pg, lane, lg);
    else if (tier == 2) page_logits_pair<2>(pg, lane, lg);
    else page_logits_pair<3>(pg, lane, lg);
    const int valid = s < 4 ? valid0 : valid1, vmax = max(valid0, valid1);
#pragma unroll
    for (int pass = 0; pass < 4; ++pass)
        if (pass * 4 + k >= valid) lg[pass] = -INFINITY;
    float pm = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
    pm = fmaxf(pm, __shfl_xor_sync(full, pm, 8));
    pm = fmaxf(pm, __shfl_xor_sync(full, pm, 16));
    const float m_new = fmaxf(st.m, pm);
    const float m_ref = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = fast_exp2(st.m - m_ref);
    st.m = m_new;
    const __half* vs = (const __half*)(pg + 2 * kP);
    float wv[4];
    bool big = false;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int t = pass * 4 + k;
        wv[pass] = t < vmax ? __half2float(vs[t]) * st.sc : 0.f;
        big |= wv[pass] > kWeightMax;
    }
    float alpha_acc = alpha;
    if (__any_sync(full, big)) {
        float vm = fmaxf(fmaxf(wv[0], wv[1]), fmaxf(wv[2], wv[3]));
        vm = fmaxf(vm, __shfl_xor_sync(full, vm, 8));
        vm = fmaxf(vm, __shfl_xor_sync(full, vm, 16));
        const float ratio = pow2_floor(kWeightMax / vm);
        st.sc *= ratio;
        alpha_acc *= ratio;
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) wv[pass] *= ratio;
    }
    float psum = 0.f;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const float pv = fast_exp2(lg[pass] - m_ref);
        psum += pv;
        pbuf[(pass * 4 + k) * kGQ2 + s] = pv * wv[pass];
    }
    st.l = st.l * alpha + psum;
    if (lane < kGQ2) pbuf[16 * kGQ2 + s] = alpha_acc;
    __syncwarp();
    page_values<kGQ2>(pg, tier, pbuf, lane, alpha_acc, st);
    __syncwarp();
}

// Output row of head hh (0 .. heads per unit - 1) of unit (b, g): query
// token q0 + hh / 4, query head 4g + hh % 4.
__device__ __forceinline__ int64_t out_row(const DecodeParams& p, int b, int g, int hh)
{
    return ((int64_t)b * p.nq + p.q0 + (hh >> 2)) * p.H_q + g * kG + (hh & 3);
}

// ------------------------------------------------------------ decode --
// NQ = 1: one query token (4 heads per unit); NQ = 2: a pair (8 heads).
template <int NQ>
__global__ void __launch_bounds__(Layout<NQ>::kWarps * 32, 1) decode_kernel(DecodeParams p)
{
    using L = Layout<NQ>;
    constexpr int kWarps = L::kWarps, kThreads = kWarps * 32, kS = L::kStages;
    constexpr int GQ = L::kHeads;   // heads per unit
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const unsigned full = 0xffffffffu;

    // Zero point of the layout: shared address 0 (absolute offsets; the
    // dynamic block must start below the first region).
    const uint32_t sbase = smem_u32(smem);
    if (sbase > L::kUpT2) {   // cannot happen with <= 8 KB of reserved shared memory
        if (tid == 0) report(p.status, SPHKV_ERR_DEVICE);
        return;
    }
    uint8_t* const Z = smem - sbase;
    constexpr uint32_t zs = 0;

    // cos/sin tables: leaf grid c*2pi/2^b_leaf, upper grid c*(pi/2)/(2^b_up-1)
    for (int e = tid; e < 2 * 256 + 64 + 16; e += kThreads) {
        double a;   // angle / pi
        uint32_t off;
        if (e < 512) {   // T1 row e/2: leaf half, upper half
            const int code = e >> 1, upper = e & 1;
            a = upper ? 0.5 * code / 255 : 2.0 * code / 256;
            off = L::kT1 + code * 256 + upper * 128;
        } else if (e < 576) {
            a = 0.5 * (e - 512) / 63;
            off = L::kUpT2 + (e - 512) * 128;
        } else {
            a = 0.5 * (e - 576) / 15;
            off = L::kUpT3 + (e - 576) * 256;
        }
        double sn, cs;
        sincospi(a, &sn, &cs);
        const float2 v = make_float2((float)cs, (float)sn);
        for (int r = 0; r < 16; ++r) ((float2*)(Z + off))[r] = v;
    }
    uint8_t* stage = Z + L::kStage + w * kS * kStageBytes;
    float* pbuf = (float*)(Z + L::kPbuf) + w * L::kPbufFloats;
    const uint32_t bar0 = zs + L::kBar + w * kS * 8;
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < kS; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_barrier_init();
    }
#ifdef SPHKV_DEBUG
    if (tid == 0) *(volatile uint32_t*)(Z + kDbgFlag<NQ>) = 0u;
#endif
    __syncthreads();

    asm volatile("griddepcontrol.wait;" ::: "memory");   // plan_kernel's results are visible
    const int32_t P = p.unit_start[p.n_units];
    const int32_t lo = cta_bound(blockIdx.x, P, p.n_cta), hi = cta_bound(blockIdx.x + 1, P, p.n_cta);
    uint32_t phase = 0;   // bit s = parity to wait for on stage s
    bool failed = false;

    float* ms_m = (float*)(Z + L::kStage);   // merge scratch, aliases the rings
    float* ms_l = ms_m + kWarps * GQ;
    float* ms_o = ms_l + kWarps * GQ;

    for (int32_t x = lo; x < hi;) {
        const int u = find_unit(p.unit_start, p.n_units, x);
        const int32_t us = p.unit_start[u], ue = p.unit_start[u + 1];
        const int32_t seg_end = min(hi, ue);
        const int b = u / p.H_kv, g = u % p.H_kv;
        const int32_t pa = x - us, pe = seg_end - us;   // unit-local page range
        const int64_t first = p.page_offsets[b];
        // tokens seen by the (first) query of this launch, and by the second
        const int len = p.seq_lens[b] - (p.nq - 1 - p.q0);
        const int len2 = p.npair == 2 ? len + 1 : 0;
        const int32_t* ptab = p.page_table + (int64_t)g * p.total_pages + first;

        // Split [pa, pe) among the warps by weight.  Warp w first sums slice w
        // (pages pa + n k / W for k = w, w + 1); after the barrier each warp
        // finds where the running weight crosses total * w / W and
        // total * (w + 1) / W.  The split depends only on the page table, so
        // results are reproducible bit for bit.
        uint32_t* wsum = (uint32_t*)(Z + L::kSlice);
        const int32_t n_seg = pe - pa;
        auto slice_start = [&](int k) -> int32_t { return pa + (int32_t)(((int64_t)n_seg * k) / kWarps); };
        {
            uint32_t sum = 0;
            for (int32_t i = slice_start(w) + lane; i < slice_start(w + 1); i += 32) sum += page_weight<NQ>(ptab[i]);
            sum = __reduce_add_sync(full, sum);
            if (lane == 0) wsum[w] = sum;
        }
        // One query: this lane's query slice in registers, q[16s .. 16s+15] of
        // the 4 heads times the logit scale, in the lane's slot order (see
        // page_logits).  Both: the unit's query-folded T2/T3 leaf tables, and
        // for a pair the T1 query rows (the previous segment ended with a
        // barrier, so no warp still reads them).  A pair launch with one query
        // (npair = 1) has heads 4-7 empty: their query is 0.
        float2 qp[kG][8];
        if constexpr (NQ == 1) {
            const int s = lane & 7, b2 = (s >> 2) & 1, b1 = (s >> 1) & 1;
#pragma unroll
            for (int i = 0; i < kG; ++i) {
                const int h = (((i >> 1) ^ b2) << 1) | ((i & 1) ^ b1);
                const float4* src = (const float4*)(p.q + out_row(p, b, g, h) * kD + 16 * s);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 v = src[k];
                    qp[i][2 * k] = make_float2(v.x * kLogitScale, v.y * kLogitScale);
                    qp[i][2 * k + 1] = make_float2(v.z * kLogitScale, v.w * kLogitScale);
                }
            }
        }
        if constexpr (NQ == 1) {
            for (int e = tid; e < 16 * kLeaves; e += kThreads) {
                const int code = e >> 6, j = e & 63, sj = j >> 3, ij = j & 7;
                const int c2 = (sj >> 2) & 1, c1 = (sj >> 1) & 1;   // slot order of the lanes owning subtree sj
                const float2 cs = *(const float2*)(Z + L::kT1 + 16 * code * 256);   // T2 code c = T1 code 16c
                float v[kG];
#pragma unroll
                for (int k = 0; k < kG; ++k) {
                    const int h = (((k >> 1) ^ c2) << 1) | ((k & 1) ^ c1);
                    const float* qh = p.q + out_row(p, b, g, h) * kD;
                    v[k] = fmaf(qh[2 * j + 1], cs.y, qh[2 * j] * cs.x) * kLogitScale;
                }
                *(float4*)(Z + L::kFold + (ij << 12) + ((uint32_t)code << 8) + (sj << 4)) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
        } else {
            // folded tables: table tb holds slots 4 tb .. 4 tb + 3 (head (4 tb + k) ^ s)
            for (int e = tid; e < 2 * 16 * kLeaves; e += kThreads) {
                const int tb = e >> 10, code = (e >> 6) & 15, j = e & 63, sj = j >> 3, ij = j & 7;
                const float2 cs = *(const float2*)(Z + L::kT1 + 16 * code * 256);
                float v[kG];
#pragma unroll
                for (int k = 0; k < kG; ++k) {
                    const int h = (4 * tb + k) ^ sj;
                    const float* qh = p.q + out_row(p, b, g, (h >> 2) < p.npair ? h : 0) * kD;
                    v[k] = (h >> 2) < p.npair ? fmaf(qh[2 * j + 1], cs.y, qh[2 * j] * cs.x) * kLogitScale : 0.f;
                }
                *(float4*)(Z + L::kFold + (ij << 12) + ((uint32_t)code << 8) + tb * L::kFold2 + (sj << 4)) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
            // T1 query rows: (q[2j], q[2j+1]) of slots 2 hp, 2 hp + 1
            for (int e = tid; e < 4 * kLeaves; e += kThreads) {
                const int hp = e >> 6, j = e & 63, sj = j >> 3, ij = j & 7;
                float v[4];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int h = (2 * hp + u) ^ sj;
                    const bool live = (h >> 2) < p.npair;
                    const float* qh = p.q + out_row(p, b, g, live ? h : 0) * kD + 2 * j;
                    v[2 * u] = live ? qh[0] * kLogitScale : 0.f;
                    v[2 * u + 1] = live ? qh[1] * kLogitScale : 0.f;
                }
                *(float4*)(Z + L::kQ + 512 * ij + 128 * hp + 16 * sj) = make_float4(v[0], v[1], v[2], v[3]);
            }
        }
        __syncthreads();
        int32_t ra, rb;   // this warp's unit-local page range
        {
            const int64_t sl = lane < kWarps ? (int64_t)wsum[lane] : 0;
            int64_t incl = sl;   // inclusive prefix over the slices
#pragma unroll
            for (int o = 1; o < kWarps; o <<= 1) {
                const int64_t y = __shfl_up_sync(full, incl, o);
                if (lane >= o) incl += y;
            }
            const int64_t W = __shfl_sync(full, incl, kWarps - 1);
            // first page whose running weight (itself included) exceeds W k / kWarps
            auto boundary = [&](int k) -> int32_t {
                if (k == 0) return pa;
                if (k == kWarps) return pe;
                const int64_t T = W * k / kWarps;
                const uint32_t over = __ballot_sync(full, lane < kWarps && incl > T);
                if (over == 0) return pe;
                const int j = __ffs(over) - 1;
                int64_t run = __shfl_sync(full, incl, j) - __shfl_sync(full, sl, j);
                const int32_t i1 = slice_start(j + 1);
                for (int32_t base = slice_start(j); base < i1; base += 32) {
                    const int32_t i = base + lane;
                    uint32_t c = i < i1 ? page_weight<NQ>(ptab[i]) : 0u;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t y = __shfl_up_sync(full, c, o);
                        if (lane >= o) c += y;
                    }
                    const uint32_t le = __ballot_sync(full, i < i1 && run + (int64_t)c <= T);
                    const int n_le = __popc(le), n_in = min(32, i1 - base);
                    if (n_le < n_in) return base + n_le;
                    run += __shfl_sync(full, c, 31);
                }
                return i1;
            };
            ra = boundary(w);
            rb = boundary(w + 1);
        }
        WarpState st;
        st.m = -INFINITY;
        st.l = 0.f;
        st.sc = kPScale;
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) st.acc[m][i] = 0.f;

        // this warp's pages: [ra, rb).  Entries are read 32 at a time.
        struct Cursor {
            int ebase;
            int32_t ent;
            uint32_t mask;
        };
        auto refill = [&](Cursor& cu) {
            const int32_t lp = ra + cu.ebase + lane;
            cu.ent = lp < rb ? ptab[lp] : 0;
            const int t = entry_tier(cu.ent);
            bool ok = t != 0;
            if (ok && entry_page(cu.ent) >= p.pool_pages[t]) {
                report(p.status, SPHKV_ERR_DATA);
                ok = false;
            }
            cu.mask = __ballot_sync(full, ok);
        };
        auto advance = [&](Cursor& cu, int32_t& lp, int32_t& e) -> bool {
            while (cu.mask == 0) {
                cu.ebase += 32;
                if (ra + cu.ebase >= rb) return false;
                refill(cu);
            }
            const int j = __ffs(cu.mask) - 1;
            cu.mask &= cu.mask - 1;
            lp = ra + cu.ebase + j;
            e = __shfl_sync(full, cu.ent, j);
            return true;
        };
        auto page_src = [&](int32_t e) -> const uint8_t* {
            const int t = entry_tier(e);
            return p.pool[t] + entry_page(e) * (int64_t)page_bytes_of(t);
        };
        auto issue = [&](int stg, int32_t e) {
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)page_bytes_of(entry_tier(e));
#ifdef SPHKV_DEBUG
                // a canary in the stage's last word, past a shorter page: the
                // copy must not reach it
                if (bytes + 4 <= (uint32_t)kStageBytes)
                    *(volatile uint32_t*)(stage + stg * kStageBytes + kStageBytes - 4) = 0x5AFEC0DEu;
#endif
                fence_proxy_async();
                mbar_expect_tx(bar0 + 8 * stg, bytes);
                bulk_g2s(smem_u32(stage + stg * kStageBytes), page_src(e), bytes, bar0 + 8 * stg);
            }
        };
        // Pages in flight: slot i of (lpq, eq, hq) is the page i places ahead
        // of the one being computed, staged in ring stage (cur + i) % kS.
        Cursor cur_c{0, 0, 0u};
        refill(cur_c);
        int32_t lpq[kS], eq[kS];
        bool hq[kS];
#pragma unroll
        for (int i = 0; i < kS; ++i) {
            lpq[i] = 0;
            eq[i] = 0;
            hq[i] = false;
        }
        hq[0] = advance(cur_c, lpq[0], eq[0]);
#pragma unroll
        for (int i = 1; i < kS - 1; ++i) hq[i] = hq[i - 1] && advance(cur_c, lpq[i], eq[i]);
        int cur = 0;
#ifdef SPHKV_TEST_HOOKS
        // warp 0 of CTA 0 alone skips its first copy and waits with a short limit
        const bool hooked = p.test_skip_copy && blockIdx.x == 0 && w == 0;
        const bool skip_first = hooked && x == lo;
#else
        constexpr bool skip_first = false;
#endif
#pragma unroll
        for (int i = 0; i < kS - 1; ++i)
            if (hq[i] && !(i == 0 && skip_first)) issue(i, eq[i]);
        while (hq[0]) {
            // the page kS - 1 ahead goes into the stage the previous page used
            hq[kS - 1] = hq[kS - 2] && advance(cur_c, lpq[kS - 1], eq[kS - 1]);
            if (hq[kS - 1]) issue(cur == 0 ? kS - 1 : cur - 1, eq[kS - 1]);
#ifdef SPHKV_TEST_HOOKS
            const bool ok = hooked ? mbar_wait<(1L << 12)>(bar0 + 8 * cur, (phase >> cur) & 1)
                                   : mbar_wait(bar0 + 8 * cur, (phase >> cur) & 1);
#else
            const bool ok = mbar_wait(bar0 + 8 * cur, (phase >> cur) & 1);
#endif
            phase ^= 1u << cur;
            if (!ok) {
                if (lane == 0) report(p.status, SPHKV_ERR_TIMEOUT);
                failed = true;
                // drain the copies still in flight, again bounded
#pragma unroll
                for (int i = 1; i < kS; ++i) {
                    if (!hq[i]) break;
                    const int sg = (cur + i) % kS;
                    mbar_wait(bar0 + 8 * sg, (phase >> sg) & 1);
                    phase ^= 1u << sg;
                }
                break;
            }
            const uint8_t* pg = stage + cur * kStageBytes;
#ifdef SPHKV_DEBUG
            if (lane == 0 && page_bytes_of(entry_tier(eq[0])) + 4 <= kStageBytes &&
                *(volatile const uint32_t*)(pg + kStageBytes - 4) != 0x5AFEC0DEu)
                *(volatile uint32_t*)(Z + kDbgFlag<NQ>) = 1u;
#endif
            const int t = entry_tier(eq[0]);
            if constexpr (NQ == 1) {
                const int valid = min(kP, len - lpq[0] * kP);
                process_page(pg, t, valid, pbuf, lane, qp, st);
            } else {
                const int v0 = max(0, min(kP, len - lpq[0] * kP)), v1 = max(0, min(kP, len2 - lpq[0] * kP));
                process_page_pair(pg, t, v0, v1, pbuf, lane, st);
            }
#pragma unroll
            for (int i = 0; i < kS - 1; ++i) {
                lpq[i] = lpq[i + 1];
                eq[i] = eq[i + 1];
                hq[i] = hq[i + 1];
            }
            hq[kS - 1] = false;
            cur = cur + 1 == kS ? 0 : cur + 1;
        }

        // ---- CTA merge of the warps' (m, l, o) for this segment
        float lt = st.l;   // lanes with the same head duplicate: sum over k only
        lt += __shfl_xor_sync(full, lt, 8);
        lt += __shfl_xor_sync(full, lt, 16);
        if constexpr (NQ == 1) {   // hi and lo weight columns (lanes c, c ^ 2) add up
#pragma unroll
            for (int m = 0; m < 8; ++m)
#pragma unroll
                for (int i = 0; i < 4; ++i) st.acc[m][i] += __shfl_xor_sync(full, st.acc[m][i], 2);
        }
        // every warp is done with its ring; a timed-out copy in any warp ends
        // the whole CTA after this segment (every warp leaves the loop together)
        failed = __syncthreads_or(failed);
        {
            const int s = lane & 7;
            // the softmax head of lane (k, s): (s >> 2) * 2 + ((s >> 1) & 1) for
            // one query (lanes s, s ^ 1 alike), s for a pair
            const int head = NQ == 1 ? (s >> 2) * 2 + ((s >> 1) & 1) : s;
            if (NQ == 1 ? (lane < 8 && !(s & 1)) : lane < GQ) {
                ms_m[w * GQ + head] = st.m;
                ms_l[w * GQ + head] = lt;
            }
            // accumulator (tile m, i): dim 16m + g + 8*(i >> 1), head 2c + (i & 1)
            const int gq = lane >> 2, cq = lane & 3;
            const float inv_sc = 1.0f / st.sc;   // exact: sc is a power of two
            if (2 * cq < GQ) {
#pragma unroll
                for (int m = 0; m < 8; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        ms_o[(w * GQ + 2 * cq + (i & 1)) * kD + 16 * m + gq + 8 * (i >> 1)] = st.acc[m][i] * inv_sc;
            }
        }
        __syncthreads();
        for (int idx = tid; idx < GQ * kD; idx += kThreads) {
            const int h = idx >> 7, dim = idx & (kD - 1);
            float M = -INFINITY;
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, ms_m[ww * GQ + h]);
            float L = 0.f, O = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int ww = 0; ww < kWarps; ++ww) {
                    const float mw = ms_m[ww * GQ + h];
                    if (mw == -INFINITY) continue;
                    const float sc = exp2f(mw - M);
                    L += ms_l[ww * GQ + h] * sc;
                    O += ms_o[(ww * GQ + h) * kD + dim] * sc;
                }
            }
            if (pa == 0 && seg_end == ue) {   // the whole unit: final result
                if ((h >> 2) < p.npair) {
                    const int64_t row = out_row(p, b, g, h);
                    p.out[row * kD + dim] = L > 0.f ? O / L : 0.f;
                    if (dim == 0) p.lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
                }
            } else {
                float* part = p.partial + ((int64_t)(blockIdx.x + u) * GQ + h) * kPartStride;
                part[4 + dim] = O;
                if (dim == 0) {
                    part[0] = M;
                    part[1] = L;
                }
            }
        }
        __syncthreads();   // scratch free before the next segment's copies
#ifdef SPHKV_DEBUG
        if (tid == 0 && *(volatile uint32_t*)(Z + kDbgFlag<NQ>)) {
            report(p.status, SPHKV_ERR_DEVICE);
            *(volatile uint32_t*)(Z + kDbgFlag<NQ>) = 0u;
        }
#endif
        x = seg_end;
        if (failed) break;
    }
}

// --------------------------------------------------------------- merge --
template <int GQ>
__global__ void __launch_bounds__(GQ * kD) merge_kernel(DecodeParams p)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");   // decode_kernel's partials are visible
    const int u = blockIdx.x;
    const int h = threadIdx.x >> 7, dim = threadIdx.x & (kD - 1);
    if ((h >> 2) >= p.npair) return;   // no such query in this launch
    const int32_t P = p.unit_start[p.n_units];
    const int32_t us = p.unit_start[u], ue = p.unit_start[u + 1];
    const int b = u / p.H_kv, g = u % p.H_kv;
    const int64_t row = out_row(p, b, g, h);
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
            M = fmaxf(M, p.partial[((int64_t)(c + u) * GQ + h) * kPartStride]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
        for (int c = c0; c <= c1; ++c) {
            if (cta_bound(c, P, p.n_cta) == cta_bound(c + 1, P, p.n_cta)) continue;
            const float* part = p.partial + ((int64_t)(c + u) * GQ + h) * kPartStride;
            if (part[0] == -INFINITY) continue;
            const float sc = exp2f(part[0] - M);
            L += part[1] * sc;
            O += part[4 + dim] * sc;
        }
    }
    p.out[row * kD + dim] = L > 0.f ? O / L : 0.f;
    if (dim == 0) p.lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

// plan, decode, merge on stream s.  decode and merge are launched as
// programmatic dependents (PDL): each may start its prologue while the kernel
// before it finishes, and waits (griddepcontrol.wait) before reading that
// kernel's results.
template <int NQ>
void launch_decode(const DecodeParams& p, cudaStream_t s)
{
    constexpr int GQ = NQ == 1 ? kG : kGQ2;
    plan_kernel<<<1, 1024, 0, s>>>(p);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.n_cta);
    cfg.blockDim = dim3(Layout<NQ>::kWarps * 32);
    cfg.dynamicSmemBytes = Layout<NQ>::kSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, decode_kernel<NQ>, p);
    cfg.gridDim = dim3(p.n_units);
    cfg.blockDim = dim3(GQ * kD);
    cfg.dynamicSmemBytes = 0;
    cudaLaunchKernelEx(&cfg, merge_kernel<GQ>, p);
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

// Workspace: unit_start [n_units + 1] | partials [n_cta + n_units][GQ][kPartStride].
size_t ws_layout(int B, int H_kv, int n_cta, int GQ, size_t* part_off)
{
    size_t n_units = (size_t)B * H_kv;
    size_t off = ((n_units + 1) * 4 + 255) / 256 * 256;
    *part_off = off;
    return off + (size_t)(n_cta + n_units) * GQ * kPartStride * 4;
}

// Argument checks shared by the decode entry points; fills everything in p
// but the query-token fields and the workspace pointers.
sphkv_status fill_params(const char* fn, const sphkv_cache* c, int32_t H_q, const float* q, float* out, float* lse,
                         int32_t* status_dev, DecodeParams& p)
{
    if (!c || !q || !out || !lse) {
        sphkv_set_error("%s: null argument", fn);
        return SPHKV_ERR_ARG;
    }
    if (c->B <= 0 || c->H_kv <= 0 || !c->page_offsets || !c->seq_lens || !c->page_table ||
        c->total_pages < 0) {
        sphkv_set_error("%s: bad cache descriptor", fn);
        return SPHKV_ERR_ARG;
    }
    if (H_q != kG * c->H_kv) {
        sphkv_set_error("%s: H_q / H_kv must be %d (got H_q=%d, H_kv=%d)", fn, kG, H_q, c->H_kv);
        return SPHKV_ERR_ARG;
    }
    if ((uintptr_t)q & 15) {
        sphkv_set_error("%s: q must be 16-byte aligned", fn);
        return SPHKV_ERR_ARG;
    }
    if ((int64_t)c->H_kv * c->total_pages > 0x7fffffffLL || (int64_t)c->B * c->H_kv > (1 << 24)) {
        sphkv_set_error("%s: cache too large for 32-bit page indices", fn);
        return SPHKV_ERR_ARG;
    }
    p = DecodeParams{};
    for (int t = 1; t <= 3; ++t) {
        p.pool[t] = c->pool[t - 1];
        p.pool_pages[t] = c->pool[t - 1] ? c->pool_pages[t - 1] : 0;
        if ((uintptr_t)c->pool[t - 1] & 15) {
            sphkv_set_error("%s: pool %d is not 16-byte aligned", fn, t);
            return SPHKV_ERR_ARG;
        }
    }
    p.n_cta = pick_ctas(c->H_kv, c->total_pages, sm_count(0));
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
    p.status = status_dev;
    p.nq = 1;
    p.q0 = 0;
    p.npair = 1;
    p.len_shift = 0;
#ifdef SPHKV_TEST_HOOKS
    const char* skip = std::getenv("SPHKV_TEST_SKIP_FIRST_COPY");
    p.test_skip_copy = skip && skip[0] && skip[0] != '0';
#endif
    return SPHKV_OK;
}

// Opt the decode kernels into their shared memory, once per device and thread.
sphkv_status ensure_smem(const char* fn)
{
    static thread_local int attr_dev = -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        sphkv_set_error("%s: no usable current device", fn);
        return SPHKV_ERR_DEVICE;
    }
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Layout<1>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Layout<2>::kSmemBytes) != cudaSuccess) {
            sphkv_set_error("%s: cannot reserve %d bytes of shared memory", fn, Layout<2>::kSmemBytes);
            return SPHKV_ERR_DEVICE;
        }
        attr_dev = dev;
    }
    return SPHKV_OK;
}

// After the launches of a call: a launch error is reported.  Debug builds also
// wait for the call's kernels (the only place the library synchronises) so
// that an execution error surfaces at the call that caused it.
sphkv_status launched(const char* fn, void* stream)
{
    cudaError_t err = cudaGetLastError();
#ifdef SPHKV_DEBUG
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
#else
    (void)stream;
#endif
    if (err != cudaSuccess) {
        sphkv_set_error("%s: launch failed: %s", fn, cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
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
    return ws_layout(B, H_kv, pick_ctas(H_kv, total_pages, sm_count(n_sm)), kG, &off);
}

extern "C" sphkv_status sphkv_decode_attention(const sphkv_cache* c, int32_t H_q, const float* q,
                                               float* out, float* lse, void* workspace,
                                               size_t ws_bytes, int32_t* status_dev, void* stream)
{
    const char* fn = "sphkv_decode_attention";
    const CallRange range(fn);
    DecodeParams p;
    sphkv_status st = fill_params(fn, c, H_q, q, out, lse, status_dev, p);
    if (st != SPHKV_OK) return st;
    if (!workspace || ((uintptr_t)workspace & 255)) {
        sphkv_set_error("%s: workspace must be non-null and 256-byte aligned", fn);
        return SPHKV_ERR_ARG;
    }
    size_t part_off;
    const size_t need = ws_layout(c->B, c->H_kv, p.n_cta, kG, &part_off);
    if (ws_bytes < need) {
        sphkv_set_error("%s: workspace %zu bytes < %zu needed", fn, ws_bytes, need);
        return SPHKV_ERR_ARG;
    }
    p.unit_start = (int32_t*)workspace;
    p.partial = (float*)((uint8_t*)workspace + part_off);
    if ((st = ensure_smem(fn)) != SPHKV_OK) return st;
    launch_decode<1>(p, (cudaStream_t)stream);
    return launched(fn, stream);
}

extern "C" size_t sphkv_decode_mq_workspace_bytes(int32_t B, int32_t H_q, int32_t H_kv, int64_t total_pages,
                                                  int32_t n_sm)
{
    (void)H_q;
    if (B <= 0 || H_kv <= 0 || total_pages < 0) return 0;
    size_t off;
    return ws_layout(B, H_kv, pick_ctas(H_kv, total_pages, sm_count(n_sm)), kGQ2, &off);
}

extern "C" sphkv_status sphkv_decode_attention_mq(const sphkv_cache* c, int32_t n_q, int32_t H_q, const float* q,
                                                  float* out, float* lse, void* workspace, size_t ws_bytes,
                                                  int32_t* status_dev, void* stream)
{
    const char* fn = "sphkv_decode_attention_mq";
    const CallRange range(fn);
    DecodeParams p;
    sphkv_status st = fill_params(fn, c, H_q, q, out, lse, status_dev, p);
    if (st != SPHKV_OK) return st;
    if (n_q < 1 || n_q > 1024) {
        sphkv_set_error("%s: n_q must be in 1..1024 (got %d)", fn, n_q);
        return SPHKV_ERR_ARG;
    }
    if (!workspace || ((uintptr_t)workspace & 255)) {
        sphkv_set_error("%s: workspace must be non-null and 256-byte aligned", fn);
        return SPHKV_ERR_ARG;
    }
    size_t part_off;
    const size_t need = ws_layout(c->B, c->H_kv, p.n_cta, kGQ2, &part_off);
    if (ws_bytes < need) {
        sphkv_set_error("%s: workspace %zu bytes < %zu needed", fn, ws_bytes, need);
        return SPHKV_ERR_ARG;
    }
    p.unit_start = (int32_t*)workspace;
    p.partial = (float*)((uint8_t*)workspace + part_off);
    if ((st = ensure_smem(fn)) != SPHKV_OK) return st;
    p.nq = n_q;
    // query tokens two at a time; the launches share the workspace in stream
    // order (each plan waits for the previous merge)
    for (int q0 = 0; q0 < n_q; q0 += 2) {
        p.q0 = q0;
        p.npair = min(2, n_q - q0);
        p.len_shift = n_q - q0 - p.npair;
        if (p.npair == 2) launch_decode<2>(p, (cudaStream_t)stream);
        else launch_decode<1>(p, (cudaStream_t)stream);
        if ((st = launched(fn, stream)) != SPHKV_OK) return st;
    }
    return SPHKV_OK;
}

// ----------------------------------------------------- no-allocation variant --
// Some callers cannot hand the library a device workspace: an engine that owns
// every byte of device memory and forbids allocation once it has started, or a
// latency-critical loop where a cudaMalloc (and the synchronisation it can
// imply) is not acceptable.  sphkv_decode_attention_noalloc serves them: the
// same plan / decode / merge kernels run with their scratch (unit page
// offsets and split-KV partials) in the file-scope array below, which every
// GPU that loads this library holds until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
}  // namespace

extern "C" sphkv_status sphkv_decode_attention_noalloc(const sphkv_cache* c, int32_t H_q, const float* q,
                                                       float* out, float* lse, int32_t* status_dev,
                                                       void* stream)
{
    const char* fn = "sphkv_decode_attention_noalloc";
    const CallRange range(fn);
    DecodeParams p;
    sphkv_status st = fill_params(fn, c, H_q, q, out, lse, status_dev, p);
    if (st != SPHKV_OK) return st;
    size_t part_off;
    const size_t need = ws_layout(c->B, c->H_kv, p.n_cta, kG, &part_off);
    if (need > kNoAllocScratchBytes) {
        sphkv_set_error("%s: this cache needs %zu bytes of scratch but the static area holds %zu; use "
                        "sphkv_decode_attention with a caller workspace",
                        fn, need, kNoAllocScratchBytes);
        return SPHKV_ERR_ARG;
    }
    // The device address of the static array, looked up with the caller's
    // device current (a host-side symbol is not a device address).  It is
    // looked up on every call, which costs no allocation and stays right after
    // a device reset or a context switch; the first call on a device also
    // loads the module there, so make that first call before any stream
    // capture.
    void* scratch = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
    if (e != cudaSuccess || !scratch) {
        sphkv_set_error("%s: cudaGetSymbolAddress failed: %s", fn, cudaGetErrorString(e));
        return SPHKV_ERR_DEVICE;
    }
    if ((st = ensure_smem(fn)) != SPHKV_OK) return st;
    p.unit_start = (int32_t*)scratch;
    p.partial = (float*)((uint8_t*)scratch + part_off);
    launch_decode<1>(p, (cudaStream_t)stream);
    return launched(fn, stream);
}
