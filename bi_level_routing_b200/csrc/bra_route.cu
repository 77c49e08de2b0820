// bra_route.cu -- routing kernels of BRA: region means, region affinities and top-k.
//
// Region-level routing ("手把手带你读懂BiFormer源码", §1.2): the mean of each region's q and k
// tokens (step 1), the affinity A = C^-1/2 qm km^T between regions (step 2) and, per row,
// the indices of the topk largest affinities (step 3).
//
// Kernel 1 streams q and k once from HBM and writes fp32 means [B, R, C] to scratch: one small
// CTA per (image, region), each thread with all its 16-byte row loads in flight at once.
// Kernel 2 computes affinity rows,
// one warp per row, and selects the top-k in registers: rounds of warp argmax for a small k,
// a shuffle bitonic network otherwise. Keys are 64-bit (order-preserving float bits, then the
// complement of the region index), which gives affinity-descending order, ties to the lower
// region and NaN after every number, deterministically.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

// ============================================================================ region means

// One CTA per (image, region), for q and k together. Thread t owns the 16-byte vectors
// v = t, t + blockDim, ... of one region row (token column v / (C / V), V channels), and for
// each it issues the loads of all hr rows of q and of k at once (up to 2 x 8 in flight), then
// sums them in row order. The CTA then sums each channel over the wr columns in order and
// divides by rs. The arithmetic is the same for every region, so regions with equal content
// get bit-identical means.
template <typename T>
__global__ void __launch_bounds__(256) region_means_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                           float *__restrict__ qm, float *__restrict__ km, int H,
                                                           int W, int C, int n_win)
{
    constexpr int V = Vec16<T>::N;
    constexpr int ROWS = 8;
    extern __shared__ float4 part4[];  // [2][wr][C] floats
    float *part = reinterpret_cast<float *>(part4);
    const int hr = H / n_win, wr = W / n_win, R = n_win * n_win;
    const int r = blockIdx.x % R;
    const int64_t b = blockIdx.x / R;
    const int ry = r / n_win, rx = r % n_win;
    const int vpt = C / V;
    const int nvec = wr * vpt;
    const int64_t row_stride = (int64_t)W * C;
    const int64_t base = ((b * H + (int64_t)ry * hr) * W + (int64_t)rx * wr) * C;

    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float aq[V], ak[V];
#pragma unroll
        for (int i = 0; i < V; ++i) aq[i] = ak[i] = 0.f;
        const T *pq = q + base + (int64_t)v * V;
        const T *pk = k + base + (int64_t)v * V;
        for (int y0 = 0; y0 < hr; y0 += ROWS) {
            const int n = min(ROWS, hr - y0);
            uint4 rq[ROWS], rk[ROWS];
#pragma unroll
            for (int u = 0; u < ROWS; ++u)
                if (u < n) {
                    rq[u] = Vec16<T>::load_raw(pq + (int64_t)(y0 + u) * row_stride);
                    rk[u] = Vec16<T>::load_raw(pk + (int64_t)(y0 + u) * row_stride);
                }
#pragma unroll
            for (int u = 0; u < ROWS; ++u)
                if (u < n) {
                    Vec16<T>::accumulate(rq[u], aq);
                    Vec16<T>::accumulate(rk[u], ak);
                }
        }
        float4 *dq = reinterpret_cast<float4 *>(part + (size_t)(v / vpt) * C + (v % vpt) * V);
        float4 *dk = reinterpret_cast<float4 *>(part + (size_t)(wr + v / vpt) * C + (v % vpt) * V);
#pragma unroll
        for (int j = 0; j < V / 4; ++j) {
            dq[j] = make_float4(aq[4 * j], aq[4 * j + 1], aq[4 * j + 2], aq[4 * j + 3]);
            dk[j] = make_float4(ak[4 * j], ak[4 * j + 1], ak[4 * j + 2], ak[4 * j + 3]);
        }
    }
    __syncthreads();
    const float rs = (float)(hr * wr);
    for (int e = threadIdx.x; e < 2 * C; e += blockDim.x) {
        const int t = e / C, c = e % C;
        float s = 0.f;
        for (int xx = 0; xx < wr; ++xx) s += part[(size_t)(t * wr + xx) * C + c];
        (t ? km : qm)[(b * R + r) * C + c] = s / rs;
    }
}

// ============================================================================ affinity + top-k

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

__device__ __forceinline__ int key_region(unsigned long long key)
{
    return (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
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

__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long x)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, off);
        x = y > x ? y : x;
    }
    return x;
}

// One CTA per (image, block of `rows` rows), one warp per row at a time. Lane l holds the keys
// of regions s = e * 32 + l, e < E (P = 32 E >= R). The image's key means (and the block's
// query means) are staged in shared memory when STAGED, rows padded to C + 4 floats so that
// lanes reading different rows hit different banks; otherwise they are read through L1.
template <int E, bool STAGED, bool ROUNDS>
__global__ void __launch_bounds__(256, 2) route_topk_kernel(const float *__restrict__ qm, const float *__restrict__ km,
                                                         int32_t *__restrict__ idx, int R, int C, int topk, int rows,
                                                         float scale)
{
    extern __shared__ float4 smem4[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int row_blocks = (R + rows - 1) / rows;
    const int b = blockIdx.x / row_blocks;
    const int r0 = (blockIdx.x % row_blocks) * rows;
    const int nrows = min(rows, R - r0);
    const int stride = STAGED ? C + 4 : C;
    const float *gkm = km + (int64_t)b * R * C;
    const float *gqm = qm + ((int64_t)b * R + r0) * C;
    const float *kbase = gkm, *qbase = gqm;
    if (STAGED) {
        // copy the key means and this block's query means into padded rows, four 16-byte
        // loads in flight per thread
        float *skm = reinterpret_cast<float *>(smem4);
        float *sqm = skm + (size_t)R * stride;
        const int c4 = C / 4;
        const int total = (R + nrows) * c4;
        for (int e0 = threadIdx.x; e0 < total; e0 += 4 * blockDim.x) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * blockDim.x;
                if (e < total) {
                    const int s = e / c4, c = (e % c4) * 4;
                    v[u] = __ldg(reinterpret_cast<const float4 *>(s < R ? gkm + s * C + c : gqm + (s - R) * C + c));
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * blockDim.x;
                if (e < total) {
                    const int s = e / c4, c = (e % c4) * 4;
                    *reinterpret_cast<float4 *>((s < R ? skm + s * stride : sqm + (s - R) * stride) + c) = v[u];
                }
            }
        }
        __syncthreads();
        kbase = skm;
        qbase = sqm;
    }
    for (int i = warp; i < nrows; i += nwarps) {
        const int r = r0 + i;
        const float *qrow = qbase + (size_t)i * stride;
        unsigned long long key[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int s = e * 32 + lane;
            key[e] = s < R ? routing_key(dot_rows(qrow, kbase + (size_t)s * stride, C) * scale, s) : 0ull;
        }
        int32_t *out = idx + ((int64_t)b * R + r) * topk;
        if (ROUNDS) {
            // topk rounds of warp argmax; the winner's key is unique (it holds the region)
            for (int j = 0; j < topk; ++j) {
                unsigned long long best = key[0];
#pragma unroll
                for (int e = 1; e < E; ++e) best = key[e] > best ? key[e] : best;
                best = warp_max_key(best);
                if (lane == 0) out[j] = key_region(best);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    if (key[e] == best) key[e] = 0ull;
            }
        } else {
            // bitonic network, descending, over position p = e * 32 + lane
#pragma unroll
            for (int size = 2; size <= 32 * E; size <<= 1) {
#pragma unroll
                for (int st = size >> 1; st > 0; st >>= 1) {
                    if (st >= 32) {
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            const int e2 = e ^ (st >> 5);
                            if (e2 > e) {
                                const bool desc = (((e * 32 + lane) & size) == 0);
                                const unsigned long long x = key[e], y = key[e2];
                                if (desc ? (x < y) : (x > y)) {
                                    key[e] = y;
                                    key[e2] = x;
                                }
                            }
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            const unsigned long long other = __shfl_xor_sync(0xffffffffu, key[e], st);
                            const bool desc = (((e * 32 + lane) & size) == 0);
                            const bool lower = (lane & st) == 0;
                            const bool keep_max = (lower == desc);
                            key[e] = keep_max ? (other > key[e] ? other : key[e]) : (other < key[e] ? other : key[e]);
                        }
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int p = e * 32 + lane;
                if (p < topk) out[p] = key_region(key[e]);
            }
        }
    }
}

// Wide rows (R > 256): one warp per row, keys in shared memory, bitonic network there.
__global__ void __launch_bounds__(256) route_topk_wide_kernel(const float *__restrict__ qm,
                                                              const float *__restrict__ km, int32_t *__restrict__ idx,
                                                              int R, int C, int topk, int P, float scale)
{
    extern __shared__ unsigned long long keys[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int row_blocks = (R + nwarps - 1) / nwarps;
    const int b = blockIdx.x / row_blocks;
    const int r = (blockIdx.x % row_blocks) * nwarps + warp;
    if (r >= R) return;
    unsigned long long *kw = keys + (size_t)warp * P;
    const float *qrow = qm + ((int64_t)b * R + r) * C;
    for (int s = lane; s < P; s += 32)
        kw[s] = s < R ? routing_key(dot_rows(qrow, km + ((int64_t)b * R + s) * C, C) * scale, s) : 0ull;
    __syncwarp();
    for (int size = 2; size <= P; size <<= 1) {
        for (int st = size >> 1; st > 0; st >>= 1) {
            for (int e = lane; e < P; e += 32) {
                const int partner = e ^ st;
                if (partner > e) {
                    const unsigned long long x = kw[e], y = kw[partner];
                    const bool desc = (e & size) == 0;
                    if (desc ? (x < y) : (x > y)) {
                        kw[e] = y;
                        kw[partner] = x;
                    }
                }
            }
            __syncwarp();
        }
    }
    int32_t *out = idx + ((int64_t)b * R + r) * topk;
    for (int j = lane; j < topk; j += 32) out[j] = key_region(kw[j]);
}

// ============================================================================ launchers

template <typename Kernel>
static cudaError_t raise_smem_limit(Kernel kernel, size_t bytes, int (&granted)[64])
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)bytes <= granted[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) granted[dev] = (int)bytes;
    return e;
}

cudaError_t launch_region_means(const void *q, const void *k, float *qm, float *km, const Geometry &g, bool bf16,
                                int num_sms, cudaStream_t stream)
{
    (void)num_sms;
    const int V = bf16 ? 8 : 4;
    const long long nvec = (long long)g.wr * (g.C / V);
    if (nvec > kMaxMeansVectors) return cudaErrorInvalidConfiguration;  // validated earlier
    int threads = (int)(((nvec + 31) / 32) * 32);
    if (threads > 256) threads = 256;
    const size_t smem = (size_t)2 * g.wr * g.C * sizeof(float);
    static int granted[2][64] = {{0}};
    cudaError_t e = bf16 ? raise_smem_limit(region_means_kernel<__nv_bfloat16>, smem, granted[0])
                         : raise_smem_limit(region_means_kernel<float>, smem, granted[1]);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)g.B * g.R;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (bf16)
        region_means_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, smem, stream>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, qm, km, g.H, g.W, g.C, g.n_win);
    else
        region_means_kernel<float><<<(unsigned)blocks, threads, smem, stream>>>((const float *)q, (const float *)k, qm,
                                                                               km, g.H, g.W, g.C, g.n_win);
    return cudaGetLastError();
}

template <int E, bool STAGED, bool ROUNDS>
static cudaError_t launch_topk_typed(const float *qm, const float *km, int32_t *idx, const Geometry &g, int rows,
                                     float scale, size_t smem, cudaStream_t stream)
{
    static int granted[64] = {0};
    cudaError_t e = raise_smem_limit(route_topk_kernel<E, STAGED, ROUNDS>, smem, granted);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)((g.R + rows - 1) / rows) * g.B;
    route_topk_kernel<E, STAGED, ROUNDS><<<(unsigned)blocks, 256, smem, stream>>>(qm, km, idx, g.R, g.C, g.topk, rows,
                                                                                  scale);
    return cudaGetLastError();
}

template <int E>
static cudaError_t launch_topk_e(const float *qm, const float *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    const float scale = (float)(1.0 / sqrt((double)g.C));
    // topk rounds of argmax cost about topk * (E + 20) instructions; the bitonic network
    // log2(P) (log2(P) + 1) / 2 stages of about 8 E.
    int lg = 5;
    while ((1 << lg) < 32 * E) ++lg;
    const long long stages = (long long)lg * (lg + 1) / 2;
    const int rounds = (long long)g.topk * (E + 20) <= stages * E * 8 ? 1 : 0;
    const int rows = g.R <= 64 ? (g.C >= 256 ? 16 : 8) : 16;
    const size_t stage_bytes = (size_t)(g.R + rows) * (g.C + 4) * sizeof(float);
    if (stage_bytes <= 100 * 1024)
        return rounds ? launch_topk_typed<E, true, true>(qm, km, idx, g, rows, scale, stage_bytes, stream)
                      : launch_topk_typed<E, true, false>(qm, km, idx, g, rows, scale, stage_bytes, stream);
    return rounds ? launch_topk_typed<E, false, true>(qm, km, idx, g, rows, scale, 0, stream)
                  : launch_topk_typed<E, false, false>(qm, km, idx, g, rows, scale, 0, stream);
}

cudaError_t launch_route_topk(const float *qm, const float *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    if (g.R <= 32) return launch_topk_e<1>(qm, km, idx, g, stream);
    if (g.R <= 64) return launch_topk_e<2>(qm, km, idx, g, stream);
    if (g.R <= 128) return launch_topk_e<4>(qm, km, idx, g, stream);
    if (g.R <= 256) return launch_topk_e<8>(qm, km, idx, g, stream);
    int P = 512;
    while (P < g.R) P <<= 1;
    int warps = (int)((48 * 1024) / ((size_t)P * 8));
    if (warps > 8) warps = 8;
    const long long blocks = (long long)((g.R + warps - 1) / warps) * g.B;
    const float scale = (float)(1.0 / sqrt((double)g.C));
    route_topk_wide_kernel<<<(unsigned)blocks, warps * 32, (size_t)warps * P * 8, stream>>>(qm, km, idx, g.R, g.C,
                                                                                             g.topk, P, scale);
    return cudaGetLastError();
}

}  // namespace bra
