// bra_route.cu -- routing kernels of BRA: region means, region affinities and top-k.
//
// Region-level routing ("手把手带你读懂BiFormer源码", §1.2): the mean of each region's q and k
// tokens (step 1), the affinity A = C^-1/2 qm km^T between regions (step 2) and, per row,
// the indices of the topk largest affinities (step 3).
//
// Kernel 1 streams q and k once from HBM with 16-byte loads and writes fp32 means [B, R, C]
// to scratch. Kernel 2 computes one affinity row per warp and selects its top-k with a
// warp-wide bitonic sort of 64-bit keys (order-preserving float bits, then the complement
// of the region index), which gives affinity-descending order, ties to the lower region and
// NaN after every number, deterministically.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

// One CTA = one band of region rows (image b, region row ry) for a chunk of region columns,
// of q (blockIdx.y == 0) or k (blockIdx.y == 1).
// Pass 1: each thread owns 16-byte vectors (one token column x, V channels) and sums them over
//         the band's hr image rows in order, into part[x][c] in shared memory.
// Pass 2: each (region, channel) sums its wr columns in order and divides by rs.
// The summation order is the same for every region, so regions with equal content get
// bit-identical means (exact affinity ties stay exact).
template <typename T>
__global__ void __launch_bounds__(256, 4) region_means_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                           float *__restrict__ qm, float *__restrict__ km, int H,
                                                           int W, int C, int n_win, int rx_per_cta, int n_chunks)
{
    extern __shared__ float4 part4[];  // [rx_per_cta * wr][C] floats
    float *part = reinterpret_cast<float *>(part4);
    constexpr int V = Vec16<T>::N;
    constexpr int ROWS = 8;  // loads in flight per thread
    const int hr = H / n_win, wr = W / n_win, R = n_win * n_win;
    const int chunk = blockIdx.x % n_chunks;
    const int band = blockIdx.x / n_chunks;
    const int ry = band % n_win, b = band / n_win;
    const int rx0 = chunk * rx_per_cta;
    const int nrx = min(rx_per_cta, n_win - rx0);
    const int ncols = nrx * wr;
    const T *x = blockIdx.y ? k : q;
    float *xm = blockIdx.y ? km : qm;

    const int vpt = C / V;  // vectors per token
    const int nvec = ncols * vpt;
    const int64_t row_stride = (int64_t)W * C;
    const T *base = x + (((int64_t)b * H + (int64_t)ry * hr) * W + (int64_t)rx0 * wr) * C;

    for (int p = threadIdx.x; p < nvec; p += blockDim.x) {
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = 0.f;
        const T *ptr = base + (int64_t)p * V;
        for (int y0 = 0; y0 < hr; y0 += ROWS) {
            const int n = min(ROWS, hr - y0);
            uint4 raw[ROWS];
#pragma unroll
            for (int u = 0; u < ROWS; ++u)
                if (u < n) raw[u] = Vec16<T>::load_raw(ptr + (int64_t)(y0 + u) * row_stride);
#pragma unroll
            for (int u = 0; u < ROWS; ++u)
                if (u < n) Vec16<T>::accumulate(raw[u], acc);
        }
        float4 *dst = reinterpret_cast<float4 *>(part + (p / vpt) * C + (p % vpt) * V);
#pragma unroll
        for (int i = 0; i < V / 4; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    }
    __syncthreads();

    const float rs = (float)(hr * wr);
    for (int e = threadIdx.x; e < nrx * C; e += blockDim.x) {
        const int j = e / C, c = e % C;
        float s = 0.f;
        for (int xx = 0; xx < wr; ++xx) s += part[(j * wr + xx) * C + c];
        xm[((int64_t)b * R + (int64_t)ry * n_win + rx0 + j) * C + c] = s / rs;
    }
}

// Order-preserving 64-bit key: larger affinity -> larger key; equal affinities -> the lower
// region gets the larger key; NaN -> below every number; 0 is below every real entry
// (used for padding).
__device__ __forceinline__ unsigned long long routing_key(float a, int s)
{
    if (a == 0.f) a = 0.f;  // -0 and +0 are equal affinities
    const uint32_t u = __float_as_uint(a);
    const uint32_t f = (a != a) ? 0u : ((u & 0x80000000u) ? ~u : (u | 0x80000000u));
    return ((unsigned long long)f << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)s);
}

// Dot product of two fp32 rows of length C (a multiple of 4) with four interleaved partial
// sums, combined in a fixed order: the same arithmetic for every row pair, so equal rows
// give equal results.
__device__ __forceinline__ float dot_rows(const float *__restrict__ a, const float *__restrict__ b, int C)
{
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    for (int c = 0; c < C; c += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(a + c);
        const float4 y = *reinterpret_cast<const float4 *>(b + c);
        s0 = fmaf(x.x, y.x, s0);
        s1 = fmaf(x.y, y.y, s1);
        s2 = fmaf(x.z, y.z, s2);
        s3 = fmaf(x.w, y.w, s3);
    }
    return (s0 + s1) + (s2 + s3);
}

// One CTA per (image, block of `rows` affinity rows); each warp handles rows in turn. The
// image's key means (and this block's query means) are staged in shared memory when
// `staged` (rows padded to C + 4 floats: lanes reading different rows hit different banks),
// otherwise read through L1. Per row, lane s computes A[r, s], the keys go to the warp's
// slice of shared memory, and a bitonic network sorts them descending.
__global__ void __launch_bounds__(256, 1) route_topk_kernel(const float *__restrict__ qm, const float *__restrict__ km,
                                                         int32_t *__restrict__ idx, int R, int C, int topk, int P,
                                                         int rows, int staged, float scale)
{
    extern __shared__ unsigned long long keys[];  // [warps][P], then staged means
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int row_blocks = (R + rows - 1) / rows;
    const int b = blockIdx.x / row_blocks;
    const int r0 = (blockIdx.x % row_blocks) * rows;
    const int nrows = min(rows, R - r0);
    const int stride = C + 4;
    float *skm = reinterpret_cast<float *>(keys + (size_t)nwarps * P);
    float *sqm = skm + (size_t)R * stride;
    const float *gkm = km + (int64_t)b * R * C;
    const float *gqm = qm + ((int64_t)b * R + r0) * C;
    if (staged) {
        for (int e = threadIdx.x; e < R * (C / 4); e += blockDim.x) {
            const int s = e / (C / 4), c = (e % (C / 4)) * 4;
            *reinterpret_cast<float4 *>(skm + s * stride + c) = __ldg(reinterpret_cast<const float4 *>(gkm + s * C + c));
        }
        for (int e = threadIdx.x; e < nrows * (C / 4); e += blockDim.x) {
            const int s = e / (C / 4), c = (e % (C / 4)) * 4;
            *reinterpret_cast<float4 *>(sqm + s * stride + c) = __ldg(reinterpret_cast<const float4 *>(gqm + s * C + c));
        }
        __syncthreads();
    }
    unsigned long long *kw = keys + (size_t)warp * P;
    for (int i = warp; i < nrows; i += nwarps) {
        const int r = r0 + i;
        const float *qrow = staged ? sqm + i * stride : gqm + i * C;
        for (int s = lane; s < P; s += 32) {
            unsigned long long key = 0ull;
            if (s < R) key = routing_key(dot_rows(qrow, staged ? skm + s * stride : gkm + s * C, C) * scale, s);
            kw[s] = key;
        }
        __syncwarp();
        for (int size = 2; size <= P; size <<= 1) {
            for (int st = size >> 1; st > 0; st >>= 1) {
                for (int e = lane; e < P; e += 32) {
                    const int partner = e ^ st;
                    if (partner > e) {
                        const unsigned long long x = kw[e], y = kw[partner];
                        const bool descending = (e & size) == 0;
                        if (descending ? (x < y) : (x > y)) {
                            kw[e] = y;
                            kw[partner] = x;
                        }
                    }
                }
                __syncwarp();
            }
        }
        int32_t *out = idx + ((int64_t)b * R + r) * topk;
        for (int j = lane; j < topk; j += 32) out[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(kw[j] & 0xFFFFFFFFull));
        __syncwarp();
    }
}

cudaError_t launch_region_means(const void *q, const void *k, float *qm, float *km, const Geometry &g, bool bf16,
                                int num_sms, cudaStream_t stream)
{
    const int elem = bf16 ? 2 : 4;
    const int V = 16 / elem;
    // Region columns per CTA: the partial sums must fit in 48 KB, and the grid should give
    // every SM several CTAs.
    int rx_per_cta = g.n_win;
    auto grid_for = [&](int rpc) { return (long long)g.B * g.n_win * ((g.n_win + rpc - 1) / rpc) * 2; };
    while (rx_per_cta > 1 &&
           ((size_t)rx_per_cta * g.wr * g.C * sizeof(float) > 48 * 1024 || grid_for(rx_per_cta) < 4LL * num_sms))
        rx_per_cta = (rx_per_cta + 1) / 2;
    const size_t smem = (size_t)rx_per_cta * g.wr * g.C * sizeof(float);
    if (smem > 48 * 1024) return cudaErrorInvalidConfiguration;  // wr * C too large (validated earlier)
    const int n_chunks = (g.n_win + rx_per_cta - 1) / rx_per_cta;
    const int nvec = rx_per_cta * g.wr * (g.C / V);
    int threads = ((nvec + 31) / 32) * 32;
    threads = threads < 64 ? 64 : (threads > 256 ? 256 : threads);
    const dim3 grid((unsigned)((long long)g.B * g.n_win * n_chunks), 2);
    if (bf16)
        region_means_kernel<__nv_bfloat16><<<grid, threads, smem, stream>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, qm, km, g.H, g.W, g.C, g.n_win, rx_per_cta, n_chunks);
    else
        region_means_kernel<float><<<grid, threads, smem, stream>>>((const float *)q, (const float *)k, qm, km, g.H,
                                                                   g.W, g.C, g.n_win, rx_per_cta, n_chunks);
    return cudaGetLastError();
}

cudaError_t launch_route_topk(const float *qm, const float *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    int P = 1;
    while (P < g.R) P <<= 1;
    if (P < 32) P = 32;
    const int warps = 8;
    const int rows = 16;
    const size_t key_bytes = (size_t)warps * P * 8;
    const size_t stage_bytes = (size_t)(g.R + rows) * (g.C + 4) * sizeof(float);
    const int staged = key_bytes + stage_bytes <= 160 * 1024;
    const size_t smem = key_bytes + (staged ? stage_bytes : 0);
    static int granted[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)smem > granted[dev]) {
        e = cudaFuncSetAttribute(route_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        granted[dev] = (int)smem;
    }
    const long long blocks = (long long)((g.R + rows - 1) / rows) * g.B;
    const float scale = (float)(1.0 / sqrt((double)g.C));
    route_topk_kernel<<<(unsigned)blocks, warps * 32, smem, stream>>>(qm, km, idx, g.R, g.C, g.topk, P, rows, staged,
                                                                      scale);
    return cudaGetLastError();
}

}  // namespace bra
