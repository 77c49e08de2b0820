// bra_attend_simt.cu -- token-to-token attention over the routed regions on CUDA cores.
//
// For every query token of region r and every head: softmax, scale head_dim^-1/2, over the
// tokens of the regions idx[b, r, 0..topk-1] (in that order, row-major inside a region),
// then the weighted sum of their values ("从零构建BiFormer", §2.2 TokenAttention;
// "医学图像分割模块：BiFormer / 双层路由注意力", §五 steps ⑤-⑦). The gathered K/V is never
// materialised: keys are read in place.
//
// One thread per (query token, head), keeping q and the running output in registers and
// folding the softmax online (running max and sum, exp2 with a log2(e) pre-scale). All
// threads of a block share (image, region, head), so their key and value loads are the
// same addresses (broadcast). This kernel serves every dtype and head size up to
// kSimtMaxHeadDim; it is the fp32 path and the fallback of the bf16 tensor-core kernels.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

template <typename T, int HDMAX>
__global__ void __launch_bounds__(128) attend_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                          const T *__restrict__ v, const int32_t *__restrict__ idx,
                                                          T *__restrict__ out, int H, int W, int C, int heads,
                                                          int n_win, int topk, float scale_log2, unsigned *err)
{
    grid_dependency_wait();
    const int hd = C / heads;
    const int hr = H / n_win, wr = W / n_win, rs = hr * wr, R = n_win * n_win;
    const int64_t blk = blockIdx.x;
    const int h = (int)(blk % heads);
    const int r = (int)((blk / heads) % R);
    const int64_t b = blk / ((int64_t)heads * R);
    const int ry = r / n_win, rx = r % n_win;
    const int32_t *routed = idx + (b * R + r) * topk;

    for (int tl = threadIdx.x; tl < rs; tl += blockDim.x) {
        const int y = ry * hr + tl / wr, x = rx * wr + tl % wr;
        const int64_t qoff = ((b * H + y) * W + x) * C + (int64_t)h * hd;
        float qv[HDMAX], o[HDMAX];
#pragma unroll
        for (int c = 0; c < HDMAX; ++c) {
            qv[c] = (c < hd) ? to_float(q[qoff + c]) : 0.f;
            o[c] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < topk; ++j) {
            const int s = routed[j];
            if (s < 0 || s >= R) {
                flag_error(err, kErrIndex);
                continue;
            }
            const int sy = s / n_win, sx = s % n_win;
            for (int kt = 0; kt < rs; ++kt) {
                const int ky = sy * hr + kt / wr, kx = sx * wr + kt % wr;
                const int64_t koff = ((b * H + ky) * W + kx) * C + (int64_t)h * hd;
                float dot = 0.f;
#pragma unroll
                for (int c = 0; c < HDMAX; ++c)
                    if (c < hd) dot = fmaf(qv[c], to_float(k[koff + c]), dot);
                const float sl = dot * scale_log2;  // logit in log2 units
                if (sl > m) {
                    const float corr = exp2f(m - sl);
                    l *= corr;
#pragma unroll
                    for (int c = 0; c < HDMAX; ++c) o[c] *= corr;
                    m = sl;
                }
                const float p = exp2f(sl - m);
                l += p;
#pragma unroll
                for (int c = 0; c < HDMAX; ++c)
                    if (c < hd) o[c] = fmaf(p, to_float(v[koff + c]), o[c]);
            }
        }
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < HDMAX; ++c)
            if (c < hd) out[qoff + c] = from_float<T>(o[c] * inv);
    }
}

template <typename T>
static cudaError_t launch_simt_typed(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                                     const Geometry &g, unsigned *err, cudaStream_t stream)
{
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    int threads = ((g.rs + 31) / 32) * 32;
    if (threads > 128) threads = 128;
    const long long blocks = (long long)g.B * g.R * g.heads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)blocks);
    const T *tq = (const T *)q, *tk = (const T *)k, *tv = (const T *)v;
    T *to = (T *)out;
    if (g.hd <= 32)
        return launch_pdl(attend_simt_kernel<T, 32>, grid, dim3(threads), 0, stream, tq, tk, tv, idx, to, g.H, g.W, g.C,
                          g.heads, g.n_win, g.topk, scale_log2, err);
    if (g.hd <= 64)
        return launch_pdl(attend_simt_kernel<T, 64>, grid, dim3(threads), 0, stream, tq, tk, tv, idx, to, g.H, g.W, g.C,
                          g.heads, g.n_win, g.topk, scale_log2, err);
    return launch_pdl(attend_simt_kernel<T, 128>, grid, dim3(threads), 0, stream, tq, tk, tv, idx, to, g.H, g.W, g.C,
                      g.heads, g.n_win, g.topk, scale_log2, err);
}

cudaError_t launch_attend_simt(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                               const Geometry &g, bool bf16, unsigned *err, cudaStream_t stream)
{
    return bf16 ? launch_simt_typed<__nv_bfloat16>(q, k, v, idx, out, g, err, stream)
                : launch_simt_typed<float>(q, k, v, idx, out, g, err, stream);
}

}  // namespace bra
