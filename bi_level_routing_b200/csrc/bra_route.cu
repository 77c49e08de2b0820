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
__global__ void __launch_bounds__(512) region_means_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                           float *__restrict__ qm, float *__restrict__ km, int H,
                                                           int W, int C, int n_win, int rx_per_cta, int n_chunks)
{
    extern __shared__ float part[];  // [rx_per_cta * wr][C]
    constexpr int V = Vec16<T>::N;
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
        int yy = 0;
        for (; yy + 4 <= hr; yy += 4) {
            float f[4][V];
#pragma unroll
            for (int u = 0; u < 4; ++u) Vec16<T>::load(ptr + (int64_t)(yy + u) * row_stride, f[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] += f[u][i];
        }
        for (; yy < hr; ++yy) {
            float f[V];
            Vec16<T>::load(ptr + (int64_t)yy * row_stride, f);
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] += f[i];
        }
        float *dst = part + (p / vpt) * C + (p % vpt) * V;
#pragma unroll
        for (int i = 0; i < V; ++i) dst[i] = acc[i];
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

// One warp per affinity row (blockIdx.x = image b * row blocks + row block). keys: P (power of two >= R)
// entries per warp in shared memory, sorted descending by a warp-wide bitonic network.
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ qm, const float *__restrict__ km,
                                                         int32_t *__restrict__ idx, int R, int C, int topk, int P,
                                                         float scale)
{
    extern __shared__ unsigned long long keys[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_blocks = (R + (blockDim.x >> 5) - 1) / (blockDim.x >> 5);
    const int b = blockIdx.x / row_blocks;
    const int r = (blockIdx.x % row_blocks) * (blockDim.x >> 5) + warp;
    if (r >= R) return;
    unsigned long long *kw = keys + (size_t)warp * P;
    const float *qrow = qm + ((int64_t)b * R + r) * C;

    for (int s = lane; s < P; s += 32) {
        unsigned long long key = 0ull;
        if (s < R) {
            const float *krow = km + ((int64_t)b * R + s) * C;
            float dot = 0.f;
            for (int c = 0; c < C; c += 4) {
                const float4 qa = __ldg(reinterpret_cast<const float4 *>(qrow + c));
                const float4 ka = __ldg(reinterpret_cast<const float4 *>(krow + c));
                dot = fmaf(qa.x, ka.x, dot);
                dot = fmaf(qa.y, ka.y, dot);
                dot = fmaf(qa.z, ka.z, dot);
                dot = fmaf(qa.w, ka.w, dot);
            }
            key = routing_key(dot * scale, s);
        }
        kw[s] = key;
    }
    __syncwarp();

    // bitonic sort, descending
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = lane; i < P; i += 32) {
                const int partner = i ^ stride;
                if (partner > i) {
                    const unsigned long long a = kw[i], c = kw[partner];
                    const bool descending = (i & size) == 0;
                    if (descending ? (a < c) : (a > c)) {
                        kw[i] = c;
                        kw[partner] = a;
                    }
                }
            }
            __syncwarp();
        }
    }

    int32_t *out = idx + ((int64_t)b * R + r) * topk;
    for (int j = lane; j < topk; j += 32) out[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(kw[j] & 0xFFFFFFFFull));
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
    threads = threads < 64 ? 64 : (threads > 512 ? 512 : threads);
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
    int warps = 8;
    while (warps > 1 && (size_t)warps * P * 8 > 48 * 1024) --warps;
    const dim3 grid((unsigned)((long long)((g.R + warps - 1) / warps) * g.B));
    const float scale = (float)(1.0 / sqrt((double)g.C));
    route_topk_kernel<<<grid, warps * 32, (size_t)warps * P * 8, stream>>>(qm, km, idx, g.R, g.C, g.topk, P, scale);
    return cudaGetLastError();
}

}  // namespace bra
