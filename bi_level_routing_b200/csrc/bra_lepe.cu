// bra_lepe.cu -- the LePE epilogue: y = x + lepe(x), lepe a 5 x 5 depthwise convolution with zero
// padding 2 and a bias per channel ("医学图像分割模块：BiFormer / 双层路由注意力", §五 step ⑧: the
// attention output viewed as a [C, H, W] image, plus nn.Conv2d(C, C, 5, padding=2, groups=C) of
// it). x and y are [B, H, W, C] (bf16 or fp32); weight is fp32 [C, 5, 5] (cross-correlation, as
// nn.Conv2d), bias fp32 [C]. Arithmetic in fp32, y rounded to the element type.
//
// One CTA per (image, 16 x 8 output tokens, block of CB channels): the 20 x 12 input tokens of the
// tile and its 2-token halo (zeros outside the image) are staged in shared memory as fp32, with
// the block's 25 taps and bias. Thread (column ox, channel pair cp) keeps the pair's 25 taps and
// the 16 outputs of its column in registers and sweeps the column's 20 input rows once, adding
// each row's 5 taps into the outputs it reaches (packed fp32 FMAs); then it adds the residual and
// writes the pairs. Every input element is read from global memory once per tile it touches
// (halo included), every output written once.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

constexpr int kTileY = 16, kTileX = 8;  // output tokens per tile
constexpr int kInY = kTileY + 4, kInX = kTileX + 4;  // input tokens per tile (halo 2)
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

// ROWS: output rows per thread, CB / 4 (CB / 2 channel pairs x kTileX columns x kTileY / ROWS row
// groups = 256 threads); a template argument, so that every loop below unrolls completely and
// every index division is by a constant.
template <typename T, int ROWS>
__global__ void __launch_bounds__(kLepeThreads) lepe_kernel(const T *__restrict__ x, const float *__restrict__ weight,
                                                            const float *__restrict__ bias, T *__restrict__ y, int H,
                                                            int W, int C)
{
    constexpr int CB = 4 * ROWS;  // channels of the CTA's block
    extern __shared__ float4 smem4[];
    float *sx = reinterpret_cast<float *>(smem4);  // [kInY * kInX][CB]
    float *sw = sx + kInY * kInX * CB;             // [25][CB]: tap-major, channels contiguous
    float *sb = sw + 25 * CB;                      // [CB]
    const int nblk = C / CB;
    const int tiles_x = (W + kTileX - 1) / kTileX, tiles_y = (H + kTileY - 1) / kTileY;
    int64_t blk = blockIdx.x;
    const int cb = (int)(blk % nblk);
    blk /= nblk;
    const int tx = (int)(blk % tiles_x);
    blk /= tiles_x;
    const int ty = (int)(blk % tiles_y);
    const int64_t b = blk / tiles_y;
    const int y0 = ty * kTileY - 2, x0 = tx * kTileX - 2, c0 = cb * CB;
    grid_dependency_wait();

    // stage the input tile with its halo (16-byte vectors of channels; four loads per thread in
    // flight before their shared-memory stores), the taps (read in their global order, which is
    // contiguous for the block: channel-major, 25 taps each) and the bias
    constexpr int V = Vec16<T>::N;
    constexpr int kBatch = 4;
    constexpr int vpt = CB / V, nvec = kInY * kInX * vpt;
    for (int e0 = threadIdx.x; e0 < nvec; e0 += kBatch * kLepeThreads) {
        uint4 raw[kBatch];
        bool inside[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int e = e0 + i * kLepeThreads;
            const int tok = e / vpt, u = e - tok * vpt;
            const int iy = y0 + tok / kInX, ix = x0 + tok % kInX;
            inside[i] = e < nvec && iy >= 0 && iy < H && ix >= 0 && ix < W;
            if (inside[i]) raw[i] = Vec16<T>::load_raw(x + ((b * H + iy) * W + ix) * C + c0 + u * V);
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int e = e0 + i * kLepeThreads;
            if (e >= nvec) break;
            float f[V];
            if (inside[i]) {
                Vec16<T>::unpack(raw[i], f);
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j) f[j] = 0.f;
            }
            const int tok = e / vpt, u = e - tok * vpt;
            float4 *d = reinterpret_cast<float4 *>(sx + tok * CB + u * V);
#pragma unroll
            for (int j = 0; j < V / 4; ++j) d[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
        }
    }
    for (int e = threadIdx.x; e < 25 * CB; e += kLepeThreads) {
        const int tap = e / CB, c = e - tap * CB;  // consecutive threads: consecutive channels of a tap
        sw[e] = weight[(int64_t)(c0 + c) * 25 + tap];
    }
    for (int c = threadIdx.x; c < CB; c += kLepeThreads) sb[c] = bias[c0 + c];
    __syncthreads();

    // thread: channel pair cp of output column ox and rows [half ROWS, (half + 1) ROWS) of the tile
    // (a CTA has CB / 2 x kTileX x kTileY / ROWS = 256 such threads)
    constexpr int pairs = CB / 2;
    const int cp = threadIdx.x % pairs, col = threadIdx.x / pairs;
    const int ox = col % kTileX, half = col / kTileX;
    const int oy0 = half * ROWS;
    float2 wt[25];
#pragma unroll
    for (int i = 0; i < 25; ++i) wt[i] = *reinterpret_cast<const float2 *>(&sw[i * CB + 2 * cp]);
    float2 acc[ROWS];
    const float2 bb = make_float2(sb[2 * cp], sb[2 * cp + 1]);
#pragma unroll
    for (int i = 0; i < ROWS; ++i) acc[i] = bb;
    // input rows oy0 .. oy0 + ROWS + 3; input row r reaches output row r - dy with tap row dy
#pragma unroll
    for (int r = 0; r < ROWS + 4; ++r) {
        float2 xr[5];
#pragma unroll
        for (int dx = 0; dx < 5; ++dx)
            xr[dx] = *reinterpret_cast<const float2 *>(&sx[((oy0 + r) * kInX + ox + dx) * CB + 2 * cp]);
#pragma unroll
        for (int dy = 0; dy < 5; ++dy) {
            if (r - dy >= 0 && r - dy < ROWS) {
#pragma unroll
                for (int dx = 0; dx < 5; ++dx) acc[r - dy] = __ffma2_rn(xr[dx], wt[dy * 5 + dx], acc[r - dy]);
            }
        }
    }
    const int gx = tx * kTileX + ox;
#pragma unroll
    for (int o = 0; o < ROWS; ++o) {
        const int oy = oy0 + o, gy = ty * kTileY + oy;
        if (gy < H && gx < W) {
            const float2 xc = *reinterpret_cast<const float2 *>(&sx[((oy + 2) * kInX + ox + 2) * CB + 2 * cp]);
            store_pair(y + ((b * H + gy) * W + gx) * C + c0 + 2 * cp, xc.x + acc[o].x, xc.y + acc[o].y);
        }
    }
}

template <typename T, int ROWS>
static cudaError_t launch_rows(const void *x, const float *weight, const float *bias, void *y, int H, int W, int C,
                               long long blocks, size_t smem, cudaStream_t stream)
{
    static int granted[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)smem > granted[dev]) {
        e = cudaFuncSetAttribute(lepe_kernel<T, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        granted[dev] = (int)smem;
    }
    return launch_pdl(lepe_kernel<T, ROWS>, dim3((unsigned)blocks), dim3(kLepeThreads), smem, stream,
                      static_cast<const T *>(x), weight, bias, static_cast<T *>(y), H, W, C);
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
    const size_t smem = ((size_t)kInY * kInX * CB + 25 * (size_t)CB + CB) * sizeof(float);
    const long long blocks = (long long)B * ((H + kTileY - 1) / kTileY) * ((W + kTileX - 1) / kTileX) * (C / CB);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // rows per thread: CB / 2 channel pairs x 8 columns x (16 / ROWS) row groups = 256 threads
    const int rows = CB * 8 * 16 / (2 * kLepeThreads);
    switch (rows) {
    case 16: return bf16 ? launch_rows<__nv_bfloat16, 16>(x, weight, bias, y, H, W, C, blocks, smem, stream)
                         : launch_rows<float, 16>(x, weight, bias, y, H, W, C, blocks, smem, stream);
    case 8: return bf16 ? launch_rows<__nv_bfloat16, 8>(x, weight, bias, y, H, W, C, blocks, smem, stream)
                        : launch_rows<float, 8>(x, weight, bias, y, H, W, C, blocks, smem, stream);
    case 4: return bf16 ? launch_rows<__nv_bfloat16, 4>(x, weight, bias, y, H, W, C, blocks, smem, stream)
                        : launch_rows<float, 4>(x, weight, bias, y, H, W, C, blocks, smem, stream);
    case 2: return bf16 ? launch_rows<__nv_bfloat16, 2>(x, weight, bias, y, H, W, C, blocks, smem, stream)
                        : launch_rows<float, 2>(x, weight, bias, y, H, W, C, blocks, smem, stream);
    case 1: return bf16 ? launch_rows<__nv_bfloat16, 1>(x, weight, bias, y, H, W, C, blocks, smem, stream)
                        : launch_rows<float, 1>(x, weight, bias, y, H, W, C, blocks, smem, stream);
    default: return cudaErrorInvalidConfiguration;
    }
}

}  // namespace bra
