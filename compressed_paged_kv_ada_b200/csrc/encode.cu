// encode.cu -- dense K/V rows -> tier pages (prefill and append).
//
// Spherical KV (arXiv 2605.18856), Abstract: ADA keeps each key in spherical
// form, as a radius and a set of compact angle codes.  The recursive-polar tree, grids and bit layout are this library's
// fixed format (see include/sphkv.h).
//
// One warp per (token, kv head).  Lane l owns dims 4l..4l+3, i.e. leaves 2l and
// 2l+1 and the level-1 node l; higher tree levels combine partial sums of
// squares with shuffles.  All angle math is fp64 with explicit _rn intrinsics
// and the file is compiled with -fmad=false, so no product is fused into an
// add and the codes match a plain fp64 reference bit for bit.
#include <cuda_bf16.h>

#include "common.cuh"

namespace sphkv {
namespace {

constexpr double kPi = 3.141592653589793;     // the double nearest pi
constexpr double kPi2 = 1.5707963267948966;   // pi / 2 (exact half of kPi)
constexpr int kEncWarps = 8;

struct EncParams {
    const void* K;
    const void* V;
    int dtype;
    const int32_t* tok_seq;
    const int32_t* tok_pos;
    int64_t n_tok;
    int B, H_kv;
    int64_t total_pages;
    const int32_t* page_offsets;
    const int32_t* page_table;
    uint8_t* pool[4];
    int64_t pool_pages[4];
    int32_t* status;
};

__device__ inline double load_elem(const void* base, int64_t idx, int dtype)
{
    if (dtype == SPHKV_DTYPE_BF16) {
        const __nv_bfloat16* p = (const __nv_bfloat16*)base;
        return (double)__bfloat162float(p[idx]);
    }
    return (double)((const float*)base)[idx];
}

// Leaf code: phi = atan2(y, x) on the periodic grid c * 2pi / 2^b.
__device__ inline int leaf_code(double x, double y, int b)
{
    if (x == 0.0 && y == 0.0) return 0;
    double phi = atan2(y, x);
    double t = rint(__ddiv_rn(__dmul_rn(phi, (double)(1 << b)), 2.0 * kPi));
    long long M = 1LL << b;
    long long c = (long long)t;
    c = ((c % M) + M) % M;
    return (int)c;
}

// Upper code: psi = atan2(|R|, |L|) on the end-inclusive grid c*(pi/2)/(2^b-1).
__device__ inline int upper_code(double ss_l, double ss_r, int b)
{
    double top = (double)((1 << b) - 1);
    double nl = sqrt(ss_l), nr = sqrt(ss_r);
    double psi = (nl == 0.0 && nr == 0.0) ? 0.0 : atan2(nr, nl);
    double t = rint(__ddiv_rn(__dmul_rn(psi, top), kPi2));
    t = fmin(fmax(t, 0.0), top);
    return (int)t;
}

// Upper code j of subtree block s (see include/sphkv.h): level-1 nodes
// 4s..4s+3, level-2 nodes 2s, 2s+1, level-3 node s, then top node s.
__device__ inline uint32_t block_up(const uint8_t* up, int s, int j)
{
    return j < 4 ? up[4 * s + j] : j < 6 ? up[32 + 2 * s + (j - 4)] : j == 6 ? up[48 + s]
                                                                            : (s < 7 ? up[56 + s] : 0u);
}

template <int T>
__device__ void pack_token(uint8_t* page, int slot, const uint8_t* sleaf, const uint8_t* sup, const int8_t* vq,
                           int lane);

template <int T>
__device__ void encode_token(const EncParams& p, int64_t i, int g, uint8_t* page, int slot,
                             uint8_t* sleaf, uint8_t* sup, int lane)
{
    constexpr TierFmt F = Tier<T>::f;
    const unsigned full = 0xffffffffu;
    int64_t row = (i * p.H_kv + g) * kD + 4 * lane;
    double k[4], v[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        k[c] = __dadd_rn(load_elem(p.K, row + c, p.dtype), 0.0);   // -0 -> +0
        v[c] = load_elem(p.V, row + c, p.dtype);
    }
    // leaves 2l, 2l+1 and level-1 node l
    double ssa = __dadd_rn(__dmul_rn(k[0], k[0]), __dmul_rn(k[1], k[1]));
    double ssb = __dadd_rn(__dmul_rn(k[2], k[2]), __dmul_rn(k[3], k[3]));
    sleaf[2 * lane] = (uint8_t)leaf_code(k[0], k[1], F.b_leaf);
    sleaf[2 * lane + 1] = (uint8_t)leaf_code(k[2], k[3], F.b_leaf);
    sup[lane] = (uint8_t)upper_code(ssa, ssb, F.b_up);
    double ss = __dadd_rn(ssa, ssb);
    // levels 2..6: node m of level l sits at lane m << (l-1)
    int base = 32;
#pragma unroll
    for (int lvl = 1, width = 16; lvl <= 5; ++lvl, width >>= 1) {
        double ssr = __shfl_down_sync(full, ss, 1 << (lvl - 1));
        if ((lane & ((2 << (lvl - 1)) - 1)) == 0) {
            int m = lane >> lvl;
            sup[base + m] = (uint8_t)upper_code(ss, ssr, F.b_up);
            ss = __dadd_rn(ss, ssr);
        }
        base += width;
    }
    // value scale: max |v| over the 128 channels
    double a = fmax(fmax(fabs(v[0]), fabs(v[1])), fmax(fabs(v[2]), fabs(v[3])));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) a = fmax(a, __shfl_xor_sync(full, a, o));
    const double Q = F.v_bits == 8 ? 127.0 : 7.0;
    __half s16 = __double2half(__ddiv_rn(a, Q));
    double s = (double)__half2float(s16);
    int q[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        double t = s == 0.0 ? 0.0 : rint(__ddiv_rn(v[c], s));
        q[c] = (int)fmin(fmax(t, -Q), Q);
    }
    __shared__ int8_t s_vq[kEncWarps][kD];
    int8_t* vq = s_vq[threadIdx.x >> 5];
#pragma unroll
    for (int c = 0; c < 4; ++c) vq[4 * lane + c] = (int8_t)q[c];
    __syncwarp();
    pack_token<T>(page, slot, sleaf, sup, vq, lane);
    if (lane == 0) {
        __half r16 = __double2half(sqrt(ss));
        ((__half*)page)[slot] = r16;
        ((__half*)(page + 2 * kP))[slot] = s16;
        if (__hisinf(r16) || __hisinf(s16)) report(p.status, SPHKV_ERR_RANGE);
    }
}

// Write one token's codes (leaf[64], upper[63] in level order) and value
// codes vq[128] (by channel) into slot `slot` of a tier-T page, in the
// format of include/sphkv.h; the radius and scale are written by the caller.
// The whole warp takes part.
template <int T>
__device__ void pack_token(uint8_t* page, int slot, const uint8_t* sleaf, const uint8_t* sup, const int8_t* vq,
                           int lane)
{
    constexpr TierFmt F = Tier<T>::f;
    // code blocks: 8 per token; lane l writes 32-bit word l of the token's blocks
    uint8_t* codes = page + F.off_codes;
    if (T == 1) {   // block s = 16 bytes: 8 leaf codes then 8 upper codes
        const int s = lane >> 2, w = lane & 3;
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int j = 4 * (w & 1) + b;
            const uint32_t code = w < 2 ? sleaf[8 * s + j] : block_up(sup, s, j);
            word |= code << (8 * b);
        }
        ((uint32_t*)codes)[slot * 32 + lane] = word;
    } else if (T == 2) {   // u32 leaf nibbles, low 32 bits of the 48-bit upper field | u16 its high bits
        if (lane < 24) {
            const int s = lane < 16 ? lane >> 1 : lane - 16;
            uint64_t uf = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) uf |= (uint64_t)block_up(sup, s, j) << (6 * j);
            if (lane < 16) {
                uint32_t word = (uint32_t)uf;
                if ((lane & 1) == 0) {
                    word = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) word |= (uint32_t)sleaf[8 * s + j] << (4 * j);
                }
                ((uint32_t*)codes)[slot * 16 + lane] = word;
            } else {
                ((uint16_t*)(codes + kP * 64))[slot * 8 + s] = (uint16_t)(uf >> 32);
            }
        }
    } else {   // u32 upper nibbles | u16 low and u8 high bits of the 24-bit leaf field
        if (lane < 8) {
            const int s = lane;
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) word |= block_up(sup, s, j) << (4 * j);
            ((uint32_t*)codes)[slot * 8 + s] = word;
        } else if (lane < 24) {
            const int s = lane < 16 ? lane - 8 : lane - 16;
            uint32_t lf = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) lf |= (uint32_t)sleaf[8 * s + j] << (3 * j);
            if (lane < 16) ((uint16_t*)(codes + kP * 32))[slot * 8 + s] = (uint16_t)lf;
            else (codes + kP * 48)[slot * 8 + s] = (uint8_t)(lf >> 16);
        }
    }
    // value row: position p holds channel v_channel_at(p); 16-byte chunks are
    // swizzled (see include/sphkv.h) so the decoder's fragment loads are
    // bank-conflict free
    uint8_t* vsec = page + F.off_v;
    if (F.v_bits == 8) {   // lane l: positions 4l..4l+3 = chunk l>>2, bytes 4(l&3)..
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) w |= ((uint32_t)(uint8_t)vq[v_channel_at(4 * lane + b)]) << (8 * b);
        const int g = lane >> 2;
        *(uint32_t*)(vsec + slot * 128 + 16 * (g ^ (slot & 6)) + 4 * (lane & 3)) = w;
    } else if (lane < 16) {   // lane l: positions 8l..8l+7 = chunk l>>1, bytes 4(l&1)..
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) w |= ((uint32_t)vq[v_channel_at(8 * lane + b)] & 15u) << (4 * b);
        const int g = lane >> 1, i = slot >> 1;
        *(uint32_t*)(vsec + i * 128 + 16 * (g ^ ((2 * i) & 6)) + 8 * (slot & 1) + 4 * (lane & 1)) = w;
    }
}

__global__ void __launch_bounds__(kEncWarps * 32) encode_kernel(EncParams p)
{
    __shared__ uint8_t s_leaf[kEncWarps][kLeaves];
    __shared__ uint8_t s_up[kEncWarps][kUpper + 1];
    int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    int64_t wg = (int64_t)blockIdx.x * kEncWarps + wib;
    if (wg >= p.n_tok * p.H_kv) return;
    int64_t i = wg / p.H_kv;
    int g = (int)(wg % p.H_kv);
    int seq = p.tok_seq[i], pos = p.tok_pos[i];
    if (seq < 0 || seq >= p.B || pos < 0) {
        if (lane == 0) report(p.status, SPHKV_ERR_DATA);
        return;
    }
    int64_t first = p.page_offsets[seq], cap = p.page_offsets[seq + 1] - first;
    if (first < 0 || (int64_t)(pos / kP) >= cap || first + pos / kP >= p.total_pages) {
        if (lane == 0) report(p.status, SPHKV_ERR_DATA);
        return;
    }
    int32_t e = p.page_table[(int64_t)g * p.total_pages + first + pos / kP];
    int t = entry_tier(e);
    if (t == 0) return;
    int64_t phys = entry_page(e);
    if (phys >= p.pool_pages[t]) {
        if (lane == 0) report(p.status, SPHKV_ERR_DATA);
        return;
    }
    uint8_t* page = p.pool[t] + phys * (int64_t)page_bytes_of(t);
    int slot = pos % kP;
    if (t == 1) encode_token<1>(p, i, g, page, slot, s_leaf[wib], s_up[wib], lane);
    else if (t == 2) encode_token<2>(p, i, g, page, slot, s_leaf[wib], s_up[wib], lane);
    else encode_token<3>(p, i, g, page, slot, s_leaf[wib], s_up[wib], lane);
}

// ------------------------------------------------------------ migrate --
// After RDR runs again (sphkv_rdr_rerun) a page may move to a coarser tier;
// its tokens are transcoded from their codes alone.  The rule (this library's
// reading; the pages give none): each angle goes to the nearest point of the
// coarser grid, computed exactly on the code integers with ties to even; the
// radius and its drop flag are kept; the values are decoded (code * scale,
// exact in fp64) and quantised again with the encoder's rule for the new
// width.  A token whose tier does not change moves unchanged.

struct MigParams {
    int B, H_kv;
    int64_t total_pages;
    const int32_t* page_offsets;
    const int32_t* seq_lens;
    const int32_t* old_table;
    const uint8_t* old_pool[4];
    int64_t old_pages[4];
    const int32_t* new_table;
    uint8_t* new_pool[4];
    int64_t new_pages[4];
    int32_t* status;
};

// Round-half-even of num / den (num >= 0, den > 0).
__device__ inline int64_t div_rne(int64_t num, int64_t den)
{
    int64_t q = num / den;
    const int64_t r = num - q * den;
    if (2 * r > den || (2 * r == den && (q & 1))) ++q;
    return q;
}

// Nearest point of the coarser periodic leaf grid (2^b_to points).
__device__ inline int leaf_to(int c, int b_from, int b_to)
{
    return (int)(div_rne((int64_t)c << b_to, (int64_t)1 << b_from) & (((int64_t)1 << b_to) - 1));
}

// Nearest point of the coarser end-inclusive upper grid (2^b_to - 1 steps).
__device__ inline int upper_to(int c, int b_from, int b_to)
{
    return (int)div_rne((int64_t)c * ((1 << b_to) - 1), (int64_t)(1 << b_from) - 1);
}

// Read slot `slot` of a tier-T page into leaf[64], up[63] (level order) and
// vq[128] (by channel); the whole warp takes part.
template <int T>
__device__ void unpack_token(const uint8_t* page, int slot, uint8_t* sleaf, uint8_t* sup, int8_t* vq, int lane)
{
    constexpr TierFmt F = Tier<T>::f;
    const uint8_t* codes = page + F.off_codes;
    if (lane < 8) {   // block s = lane
        const int s = lane, blk = slot * 8 + s;
        uint32_t L[8], U[8];
        if (T == 1) {
            const uint8_t* b = codes + blk * 16;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                L[j] = b[j];
                U[j] = b[8 + j];
            }
        } else if (T == 2) {
            const uint64_t a = *(const uint64_t*)(codes + blk * 8);
            const uint64_t uf = (a >> 32) | ((uint64_t)*(const uint16_t*)(codes + kP * 64 + blk * 2) << 32);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                L[j] = (uint32_t)(a >> (4 * j)) & 15u;
                U[j] = (uint32_t)(uf >> (6 * j)) & 63u;
            }
        } else {
            const uint32_t u = *(const uint32_t*)(codes + blk * 4);
            const uint32_t lf = *(const uint16_t*)(codes + kP * 32 + blk * 2) | ((uint32_t)codes[kP * 48 + blk] << 16);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                U[j] = (u >> (4 * j)) & 15u;
                L[j] = (lf >> (3 * j)) & 7u;
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) sleaf[8 * s + j] = (uint8_t)L[j];
#pragma unroll
        for (int j = 0; j < 4; ++j) sup[4 * s + j] = (uint8_t)U[j];
        sup[32 + 2 * s] = (uint8_t)U[4];
        sup[32 + 2 * s + 1] = (uint8_t)U[5];
        sup[48 + s] = (uint8_t)U[6];
        if (s < 7) sup[56 + s] = (uint8_t)U[7];
    }
    const uint8_t* vsec = page + F.off_v;
    if (F.v_bits == 8) {
        const int g = lane >> 2;
        const uint32_t w = *(const uint32_t*)(vsec + slot * 128 + 16 * (g ^ (slot & 6)) + 4 * (lane & 3));
#pragma unroll
        for (int b = 0; b < 4; ++b) vq[v_channel_at(4 * lane + b)] = (int8_t)(w >> (8 * b));
    } else if (lane < 16) {
        const int g = lane >> 1, i = slot >> 1;
        const uint32_t w =
            *(const uint32_t*)(vsec + i * 128 + 16 * (g ^ ((2 * i) & 6)) + 8 * (slot & 1) + 4 * (lane & 1));
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            int x = (int)((w >> (4 * b)) & 15u);
            vq[v_channel_at(8 * lane + b)] = (int8_t)(x >= 8 ? x - 16 : x);   // two's complement nibble
        }
    }
}

template <int TF>
__device__ void unpack_any(int tf, const uint8_t* page, int slot, uint8_t* sleaf, uint8_t* sup, int8_t* vq, int lane)
{
    if (tf == 1) unpack_token<1>(page, slot, sleaf, sup, vq, lane);
    else if (tf == 2) unpack_token<2>(page, slot, sleaf, sup, vq, lane);
    else unpack_token<3>(page, slot, sleaf, sup, vq, lane);
}

__device__ inline int bits_leaf(int t) { return t == 1 ? 8 : t == 2 ? 4 : 3; }
__device__ inline int bits_up(int t) { return t == 1 ? 8 : t == 2 ? 6 : 4; }

__global__ void __launch_bounds__(kEncWarps * 32) migrate_kernel(MigParams p)
{
    __shared__ uint8_t s_leaf[kEncWarps][kLeaves];
    __shared__ uint8_t s_up[kEncWarps][kUpper + 1];
    __shared__ int8_t s_vq[kEncWarps][kD];
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t per_head = p.total_pages * kP;
    const int64_t wg = (int64_t)blockIdx.x * kEncWarps + wib;   // (kv head, logical page, slot)
    if (wg >= per_head * p.H_kv) return;
    const int g = (int)(wg / per_head);
    const int64_t lp = (wg % per_head) / kP;
    const int slot = (int)(wg % kP);
    int lo = 0, hi = p.B - 1;   // sequence owning logical page lp
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.page_offsets[mid] <= lp) lo = mid;
        else hi = mid - 1;
    }
    if (lp >= p.page_offsets[lo + 1]) return;
    if ((lp - p.page_offsets[lo]) * kP + slot >= p.seq_lens[lo]) return;   // no token in this slot
    const int32_t eo = p.old_table[(int64_t)g * p.total_pages + lp], en = p.new_table[(int64_t)g * p.total_pages + lp];
    const int to = entry_tier(eo), tn = entry_tier(en);
    if (tn == 0) return;
    if (to == 0 || tn < to || entry_page(eo) >= p.old_pages[to] || entry_page(en) >= p.new_pages[tn]) {
        if (lane == 0) report(p.status, SPHKV_ERR_DATA);   // a page cannot become finer or come back
        return;
    }
    const uint8_t* src = p.old_pool[to] + entry_page(eo) * (int64_t)page_bytes_of(to);
    uint8_t* dst = p.new_pool[tn] + entry_page(en) * (int64_t)page_bytes_of(tn);
    uint8_t* sleaf = s_leaf[wib];
    uint8_t* sup = s_up[wib];
    int8_t* vq = s_vq[wib];
    unpack_any<0>(to, src, slot, sleaf, sup, vq, lane);
    __syncwarp();
    uint16_t s16 = ((const uint16_t*)(src + 2 * kP))[slot];
    if (tn != to) {
        for (int j = lane; j < kLeaves; j += 32) sleaf[j] = (uint8_t)leaf_to(sleaf[j], bits_leaf(to), bits_leaf(tn));
        for (int j = lane; j < kUpper; j += 32) sup[j] = (uint8_t)upper_to(sup[j], bits_up(to), bits_up(tn));
        const double sa = (double)__half2float(__ushort_as_half(s16));
        double v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = __dmul_rn((double)vq[4 * lane + c], sa);
        double a = fmax(fmax(fabs(v[0]), fabs(v[1])), fmax(fabs(v[2]), fabs(v[3])));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) a = fmax(a, __shfl_xor_sync(full, a, o));
        const double Q = tn == 1 ? 127.0 : 7.0;
        const __half sb = __double2half(__ddiv_rn(a, Q));
        const double sv = (double)__half2float(sb);
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const double t = sv == 0.0 ? 0.0 : rint(__ddiv_rn(v[c], sv));
            vq[4 * lane + c] = (int8_t)fmin(fmax(t, -Q), Q);
        }
        s16 = __half_as_ushort(sb);
        if (lane == 0 && __hisinf(sb)) report(p.status, SPHKV_ERR_RANGE);
    }
    __syncwarp();
    if (tn == 1) pack_token<1>(dst, slot, sleaf, sup, vq, lane);
    else if (tn == 2) pack_token<2>(dst, slot, sleaf, sup, vq, lane);
    else pack_token<3>(dst, slot, sleaf, sup, vq, lane);
    if (lane == 0) {
        ((uint16_t*)dst)[slot] = ((const uint16_t*)src)[slot];   // radius and drop flag unchanged
        ((uint16_t*)(dst + 2 * kP))[slot] = s16;
    }
}

}  // namespace
}  // namespace sphkv

using namespace sphkv;

extern "C" sphkv_status sphkv_migrate(const sphkv_cache* from, const sphkv_cache* to, int32_t* status_dev,
                                      void* stream)
{
    const char* fn = "sphkv_migrate";
    const CallRange range(fn);
    if (!from || !to) {
        sphkv_set_error("%s: null argument", fn);
        return SPHKV_ERR_ARG;
    }
    if (from->B <= 0 || from->H_kv <= 0 || from->total_pages < 0 || !from->page_offsets || !from->seq_lens ||
        !from->page_table || !to->page_table || from->B != to->B || from->H_kv != to->H_kv ||
        from->total_pages != to->total_pages) {
        sphkv_set_error("%s: the two cache descriptors must describe the same sequences and pages", fn);
        return SPHKV_ERR_ARG;
    }
    if ((int64_t)from->H_kv * from->total_pages * kP / kEncWarps > 0x7fffffffLL) {
        sphkv_set_error("%s: cache too large", fn);
        return SPHKV_ERR_ARG;
    }
    MigParams p{};
    p.B = from->B;
    p.H_kv = from->H_kv;
    p.total_pages = from->total_pages;
    p.page_offsets = from->page_offsets;
    p.seq_lens = from->seq_lens;
    p.old_table = from->page_table;
    p.new_table = to->page_table;
    for (int t = 1; t <= 3; ++t) {
        p.old_pool[t] = from->pool[t - 1];
        p.old_pages[t] = from->pool[t - 1] ? from->pool_pages[t - 1] : 0;
        p.new_pool[t] = to->pool[t - 1];
        p.new_pages[t] = to->pool[t - 1] ? to->pool_pages[t - 1] : 0;
    }
    p.status = status_dev;
    const int64_t warps = from->H_kv * from->total_pages * kP;
    if (warps == 0) return SPHKV_OK;
    migrate_kernel<<<(unsigned)((warps + kEncWarps - 1) / kEncWarps), kEncWarps * 32, 0, (cudaStream_t)stream>>>(p);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("%s: launch failed: %s", fn, cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}

extern "C" sphkv_status sphkv_encode(const sphkv_cache* c, const void* K, const void* V, int dtype,
                                     const int32_t* tok_seq, const int32_t* tok_pos, int64_t n_tok,
                                     int32_t* status_dev, void* stream)
{
    const CallRange range("sphkv_encode");
    if (!c || (n_tok > 0 && (!K || !V || !tok_seq || !tok_pos))) {
        sphkv_set_error("sphkv_encode: null argument");
        return SPHKV_ERR_ARG;
    }
    if (dtype != SPHKV_DTYPE_F32 && dtype != SPHKV_DTYPE_BF16) {
        sphkv_set_error("sphkv_encode: dtype must be SPHKV_DTYPE_F32 or SPHKV_DTYPE_BF16");
        return SPHKV_ERR_ARG;
    }
    if (c->B <= 0 || c->H_kv <= 0 || c->total_pages < 0 || !c->page_offsets || !c->page_table) {
        sphkv_set_error("sphkv_encode: bad cache descriptor");
        return SPHKV_ERR_ARG;
    }
    if (n_tok < 0) {
        sphkv_set_error("sphkv_encode: n_tok < 0");
        return SPHKV_ERR_ARG;
    }
    if (n_tok == 0) return SPHKV_OK;
    EncParams p{};
    p.K = K;
    p.V = V;
    p.dtype = dtype;
    p.tok_seq = tok_seq;
    p.tok_pos = tok_pos;
    p.n_tok = n_tok;
    p.B = c->B;
    p.H_kv = c->H_kv;
    p.total_pages = c->total_pages;
    p.page_offsets = c->page_offsets;
    p.page_table = c->page_table;
    for (int t = 1; t <= 3; ++t) {
        p.pool[t] = c->pool[t - 1];
        p.pool_pages[t] = c->pool[t - 1] ? c->pool_pages[t - 1] : 0;
        if (c->pool[t - 1] && ((uintptr_t)c->pool[t - 1] & 15)) {
            sphkv_set_error("sphkv_encode: pool %d is not 16-byte aligned", t);
            return SPHKV_ERR_ARG;
        }
    }
    p.status = status_dev;
    int64_t warps = n_tok * c->H_kv;
    int64_t blocks = (warps + kEncWarps - 1) / kEncWarps;
    if (blocks > 0x7fffffffLL) {
        sphkv_set_error("sphkv_encode: too many rows");
        return SPHKV_ERR_ARG;
    }
    encode_kernel<<<(unsigned)blocks, kEncWarps * 32, 0, (cudaStream_t)stream>>>(p);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("sphkv_encode: launch failed: %s", cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}
