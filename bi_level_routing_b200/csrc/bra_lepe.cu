// bra_lepe.cu -- the LePE epilogue: y = x + lepe(x), lepe a 5 x 5 depthwise convolution with zero
// padding 2 and a bias per channel ("医学图像分割模块：BiFormer / 双层路由注意力", §五 step ⑧: the
// attention output viewed as a [C, H, W] image, plus nn.Conv2d(C, C, 5, padding=2, groups=C) of
// it). x and y are [B, H, W, C] (bf16 or fp32); weight is fp32 [C, 5, 5] (cross-correlation, as
// nn.Conv2d), bias fp32 [C]. Arithmetic in fp32, y rounded to the element type.
//
// One CTA per (image, 8 x 8 output tokens, block of CB channels): the 12 x 12 input tokens of the
// tile and its 2-token halo (zeros outside the image) are staged in shared memory as fp32, with
// the block's 25 taps and bias; each thread then computes a pair of channels of several output
// tokens with packed fp32 FMAs, adds the residual and writes the pair. Every input element is
// read from global memory once per tile it touches (1.0 + halo), every output written once.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

constexpr int kTile = 8;                // output tokens per tile side
constexpr int kIn = kTile + 4;          // input tokens per tile side (halo 2)
constexpr int kLepeThreads = 256;

// Two adjacent outputs (an even channel and the next) in one store: bf16 rounded to nearest even.
__device__ __forceinline__ void store_pair(__nv_bfloat16 *dst, float a, float b)
{
    *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(a, b);
}
__device__ __forceinline__ void store_pair(float *dst, float a, float b)
{
    *reinterpret_cast<float2 *>(dst) = make_float2(a, b);
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kLepeThreads) lepe_kernel(const T *__restrict__ x, const float *__restrict__ weight,
                                                            const float *__restrict__ bias, T *__restrict__ y, int H,
                                                            int W, int C, int CB)
{
    extern __shared__ float4 smem4[];
    float *sx = reinterpret_cast<float *>(smem4);  // [kIn * kIn][CB]
    float *sw = sx + kIn * kIn * CB;               // [25][CB]: tap-major, channels contiguous
    float *sb = sw + 25 * CB;                      // [CB]
    const int nblk = C / CB;
    const int tiles_x = (W + kTile - 1) / kTile, tiles_y = (H + kTile - 1) / kTile;
    int64_t blk = blockIdx.x;
    const int cb = (int)(blk % nblk);
    blk /= nblk;
    const int tx = (int)(blk % tiles_x);
    blk /= tiles_x;
    const int ty = (int)(blk % tiles_y);
    const int64_t b = blk / tiles_y;
    const int y0 = ty * kTile - 2, x0 = tx * kTile - 2, c0 = cb * CB;
    grid_dependency_wait();

    // stage the input tile with its halo (16-byte vectors of channels), the taps and the bias
    constexpr int V = Vec16<T>::N;
    const int vpt = CB / V;
    for (int e = threadIdx.x; e < kIn * kIn * vpt; e += kLepeThreads) {
        const int tok = e / vpt, u = e - tok * vpt;
        const int iy = y0 + tok / kIn, ix = x0 + tok % kIn;
        float f[V];
        if (iy >= 0 && iy < H && ix >= 0 && ix < W) {
            Vec16<T>::load(x + ((b * H + iy) * W + ix) * C + c0 + u * V, f);
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i) f[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < V; ++i) sx[tok * CB + u * V + i] = f[i];
    }
    for (int e = threadIdx.x; e < 25 * CB; e += kLepeThreads) {
        const int tap = e / CB, c = e - tap * CB;
        sw[e] = weight[(int64_t)(c0 + c) * 25 + tap];
    }
    for (int c = threadIdx.x; c < CB; c += kLepeThreads) sb[c] = bias[c0 + c];
    __syncthreads();

    // thread: channel pair cp, output tokens tg, tg + groups, ...
    const int pairs = CB / 2;
    const int cp = threadIdx.x % pairs, groups = kLepeThreads / pairs;
    const int tg = threadIdx.x / pairs;
    if (tg >= groups) return;
    const float2 bb = make_float2(sb[2 * cp], sb[2 * cp + 1]);
    for (int t = tg; t < kTile * kTile; t += groups) {
        const int oy = t / kTile, ox = t % kTile;
        const int gy = ty * kTile + oy, gx = tx * kTile + ox;
        if (gy >= H || gx >= W) continue;
        float2 acc = bb;
#pragma unroll
        for (int dy = 0; dy < 5; ++dy)
#pragma unroll
            for (int dx = 0; dx < 5; ++dx) {
                const float2 xv = *reinterpret_cast<const float2 *>(&sx[((oy + dy) * kIn + ox + dx) * CB + 2 * cp]);
                const float2 wv = *reinterpret_cast<const float2 *>(&sw[(dy * 5 + dx) * CB + 2 * cp]);
                acc = __ffma2_rn(xv, wv, acc);
            }
        const float2 xc = *reinterpret_cast<const float2 *>(&sx[((oy + 2) * kIn + ox + 2) * CB + 2 * cp]);
        const float r0 = xc.x + acc.x, r1 = xc.y + acc.y;
        store_pair(y + ((b * H + gy) * W + gx) * C + c0 + 2 * cp, r0, r1);
    }
}

bool lepe_supports(int C, bool bf16) { return C % (bf16 ? 8 : 4) == 0; }

cudaError_t launch_lepe(const void *x, const float *weight, const float *bias, void *y, int B, int H, int W, int C,
                        bool bf16, cudaStream_t stream)
{
    // channels per CTA: the largest of 64, 32, 16, 8, 4 that divides C (a whole number of
    // 16-byte vectors)
    int CB = 64;
    while (CB > 4 && C % CB != 0) CB >>= 1;
    if (C % CB != 0 || CB % (bf16 ? 8 : 4) != 0) return cudaErrorInvalidConfiguration;
    const size_t smem = ((size_t)kIn * kIn * CB + 25 * (size_t)CB + CB) * sizeof(float);
    const long long blocks = (long long)B * ((H + kTile - 1) / kTile) * ((W + kTile - 1) / kTile) * (C / CB);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (bf16)
        return launch_pdl(lepe_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(kLepeThreads), smem, stream,
                          static_cast<const __nv_bfloat16 *>(x), weight, bias, static_cast<__nv_bfloat16 *>(y), H, W,
                          C, CB);
    return launch_pdl(lepe_kernel<float>, dim3((unsigned)blocks), dim3(kLepeThreads), smem, stream,
                      static_cast<const float *>(x), weight, bias, static_cast<float *>(y), H, W, C, CB);
}

}  // namespace bra
