// splitkv.cu -- combine decode results computed over disjoint parts of the
// same sequences, e.g. one long stream whose pages are split across GPUs.
//
// Spherical KV (arXiv 2605.18856), Abstract: the decode path targets
// long-context inference.  Each part is an ordinary decode result over its
// own keys (out normalised, lse the natural-log log-sum-exp of its logits);
// with M = max_r lse_r and w_r = exp(lse_r - M) the union's result is
// out = sum_r w_r out_r / sum_r w_r and lse = M + ln sum_r w_r, the same
// combine the decode kernel uses to merge its own split-KV pieces.
#include "common.cuh"

namespace sphkv {
namespace {

// One 128-thread CTA per row (query head of a sequence), one thread per dim.
__global__ void __launch_bounds__(kD) merge_parts_kernel(const float* out_parts, const float* lse_parts,
                                                         int n_parts, int64_t n_rows, float* out, float* lse)
{
    const int d = threadIdx.x;
    for (int64_t row = blockIdx.x; row < n_rows; row += gridDim.x) {
        float M = -INFINITY;
        for (int r = 0; r < n_parts; ++r) M = fmaxf(M, lse_parts[(int64_t)r * n_rows + row]);
        float Z = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int r = 0; r < n_parts; ++r) {
                const float l = lse_parts[(int64_t)r * n_rows + row];
                if (l == -INFINITY) continue;   // a part with no kept token
                const float w = expf(l - M);
                Z += w;
                O += w * out_parts[((int64_t)r * n_rows + row) * kD + d];
            }
        }
        out[row * kD + d] = Z > 0.f ? O / Z : 0.f;
        if (d == 0) lse[row] = Z > 0.f ? M + logf(Z) : -INFINITY;
    }
}

}  // namespace
}  // namespace sphkv

using namespace sphkv;

extern "C" sphkv_status sphkv_merge_partials(const float* out_parts, const float* lse_parts, int32_t n_parts,
                                             int64_t n_rows, float* out, float* lse, void* stream)
{
    const char* fn = "sphkv_merge_partials";
    const CallRange range(fn);
    if (n_rows < 0 || n_parts < 1 || n_parts > 4096) {
        sphkv_set_error("%s: need 1 <= n_parts <= 4096 and n_rows >= 0 (got %d, %lld)", fn, n_parts,
                        (long long)n_rows);
        return SPHKV_ERR_ARG;
    }
    if (n_rows == 0) return SPHKV_OK;
    if (!out_parts || !lse_parts || !out || !lse) {
        sphkv_set_error("%s: null argument", fn);
        return SPHKV_ERR_ARG;
    }
    const int64_t grid = n_rows < (1 << 20) ? n_rows : (1 << 20);
    merge_parts_kernel<<<(unsigned)grid, kD, 0, (cudaStream_t)stream>>>(out_parts, lse_parts, n_parts, n_rows,
                                                                       out, lse);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        sphkv_set_error("%s: launch failed: %s", fn, cudaGetErrorString(err));
        return SPHKV_ERR_DEVICE;
    }
    return SPHKV_OK;
}
