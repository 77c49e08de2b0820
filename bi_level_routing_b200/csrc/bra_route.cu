// bra_route.cu -- routing kernels of BRA: region means, region affinities and top-k.
//
// Region-level routing ("手把手带你读懂BiFormer源码", §1.2): the mean of each region's q and k
// tokens (step 1), the affinity A = C^-1/2 qm km^T between regions (step 2) and, per row,
// the indices of the topk largest affinities (step 3).
//
// The means kernel streams q and k once from HBM and writes fp32 means [B, R, C] to scratch:
// a group of threads per (image, region), each thread with its 16-byte row loads in flight at
// once. The routing kernel computes affinity rows, several rows per warp pass, and selects the
// top-k in registers: rounds of warp argmax for a small k, a shuffle bitonic network otherwise. Keys are 64-bit
// (order-preserving float bits, then the complement of the region index), which gives
// affinity-descending order, ties to the lower region and NaN after every number,
// deterministically. One-token regions skip the means: the routing kernels read q and k
// themselves, and in bf16 (up to 64 regions) a tensor-core kernel forms the dot products.
#include <type_traits>

#include "bra_device.cuh"
#include "bra_launch.h"
#include "bra_routing.cuh"

namespace bra {

// ============================================================================ region means

// Arguments of the means kernel.
struct MeansArgs {
    const void *q, *k;
    float *qm, *km;
    int B, H, W, C, n_win, hr, wr, R;
    int slots;  // threads per region: the row segment's vectors rounded up to a warp, <= 256
    int rpc;    // regions per CTA (256 / slots)
};

constexpr int kMeansThreads = 256;

// The means of the regions i0 .. i0 + nreg - 1 (flat index b * R + r), q and k together. A
// region row segment is nvec = wr C / V 16-byte vectors; thread t of group g = t / slots owns
// the vectors v = t % slots, t % slots + slots, ... of region i0 + g and, eight region rows at
// a time, issues the loads of those rows of q and of k at once (16 in flight), then sums them
// in row order. The CTA then sums each channel over the wr columns in order and divides by
// rs: the arithmetic is the same for every region, so regions with equal content get
// bit-identical means.
template <typename T>
__device__ __forceinline__ void region_means_block(const MeansArgs &a, float *part, long long i0, int nreg)
{
    constexpr int V = Vec16<T>::N;
    constexpr int ROWS = 8;
    const int C = a.C;
    const int vpt = C / V;
    const int nvec = a.wr * vpt;
    const int grp = threadIdx.x / a.slots;
    if (grp < nreg) {
        const int flat = (int)i0 + grp;  // B * R < 2^31 (checked by the launcher)
        const int b = flat / a.R;
        const int r = flat - b * a.R;
        const int ry = r / a.n_win, rx = r % a.n_win;
        const int64_t row_stride = (int64_t)a.W * C;
        const int64_t base = (((int64_t)b * a.H + (int64_t)ry * a.hr) * a.W + (int64_t)rx * a.wr) * C;
        for (int v = threadIdx.x - grp * a.slots; v < nvec; v += a.slots) {
            float aq[V], ak[V];
#pragma unroll
            for (int i = 0; i < V; ++i) aq[i] = ak[i] = 0.f;
            const T *pq = static_cast<const T *>(a.q) + base + (int64_t)v * V;
            const T *pk = static_cast<const T *>(a.k) + base + (int64_t)v * V;
            for (int y0 = 0; y0 < a.hr; y0 += ROWS) {
                const int n = min(ROWS, a.hr - y0);
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
            float4 *dq = reinterpret_cast<float4 *>(part + ((size_t)(2 * grp) * a.wr + v / vpt) * C + (v % vpt) * V);
            float4 *dk = reinterpret_cast<float4 *>(part + ((size_t)(2 * grp + 1) * a.wr + v / vpt) * C + (v % vpt) * V);
#pragma unroll
            for (int j = 0; j < V / 4; ++j) {
                dq[j] = make_float4(aq[4 * j], aq[4 * j + 1], aq[4 * j + 2], aq[4 * j + 3]);
                dk[j] = make_float4(ak[4 * j], ak[4 * j + 1], ak[4 * j + 2], ak[4 * j + 3]);
            }
        }
    }
    __syncthreads();
    const float rs = (float)(a.hr * a.wr);
    for (int e = threadIdx.x; e < nreg * 2 * C; e += blockDim.x) {
        const int qc = e / C, g = qc >> 1, t = qc & 1, c = e - qc * C;
        float s = 0.f;
        for (int xx = 0; xx < a.wr; ++xx) s += part[((size_t)(2 * g + t) * a.wr + xx) * C + c];
        (t ? a.km : a.qm)[(i0 + g) * C + c] = s / rs;
    }
}

// Small regions (rs <= 16): one CTA per region. `lanes` consecutive threads per 16-byte vector
// of channels (lanes = hr when hr is 2, 4 or 8, else 1); thread j of a vector sums region rows
// j, j + lanes, ... token by token in order, with up to 4 tokens' loads of q and of k in flight,
// then a butterfly over the lanes adds the row sums in a fixed order. No shared memory, no
// barrier, and no division per token.
template <typename T>
__device__ __forceinline__ void region_means_small(const MeansArgs &a, int64_t b, int r, int lshift)
{
    constexpr int V = Vec16<T>::N;
    constexpr int TOK = 4;
    const int lanes = 1 << lshift;
    const int j = threadIdx.x & (lanes - 1);
    const int vpt = a.C / V;
    const int ry = r / a.n_win, rx = r % a.n_win;
    const int64_t base = ((b * a.H + (int64_t)ry * a.hr) * a.W + (int64_t)rx * a.wr) * a.C;
    const int64_t row_stride = (int64_t)a.W * a.C;
    const float n = (float)(a.hr * a.wr);
    const int step = blockDim.x >> lshift;
    // the same trip count for every lane of a warp, so that all of them take part in the
    // butterfly; a lane past the last vector loads and stores nothing
    for (int v0 = 0; v0 < vpt; v0 += step) {
        const int v = v0 + (threadIdx.x >> lshift);
        const bool live = v < vpt;
        const T *pq = static_cast<const T *>(a.q) + base + (int64_t)(live ? v : 0) * V;
        const T *pk = static_cast<const T *>(a.k) + base + (int64_t)(live ? v : 0) * V;
        float aq[V], ak[V];
#pragma unroll
        for (int i = 0; i < V; ++i) aq[i] = ak[i] = 0.f;
        for (int y = j; live && y < a.hr; y += lanes) {
            const T *rq0 = pq + (int64_t)y * row_stride, *rk0 = pk + (int64_t)y * row_stride;
            for (int x0 = 0; x0 < a.wr; x0 += TOK) {
                uint4 rq[TOK], rk[TOK];
#pragma unroll
                for (int u = 0; u < TOK; ++u)
                    if (x0 + u < a.wr) {
                        rq[u] = Vec16<T>::load_raw(rq0 + (int64_t)(x0 + u) * a.C);
                        rk[u] = Vec16<T>::load_raw(rk0 + (int64_t)(x0 + u) * a.C);
                    }
#pragma unroll
                for (int u = 0; u < TOK; ++u)
                    if (x0 + u < a.wr) {
                        Vec16<T>::accumulate(rq[u], aq);
                        Vec16<T>::accumulate(rk[u], ak);
                    }
            }
        }
        for (int off = 1; off < lanes; off <<= 1) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                aq[i] += __shfl_xor_sync(0xffffffffu, aq[i], off);
                ak[i] += __shfl_xor_sync(0xffffffffu, ak[i], off);
            }
        }
        if (live && j == 0) {
            float4 *dq = reinterpret_cast<float4 *>(a.qm + (b * a.R + r) * a.C + v * V);
            float4 *dk = reinterpret_cast<float4 *>(a.km + (b * a.R + r) * a.C + v * V);
#pragma unroll
            for (int i = 0; i < V / 4; ++i) {
                dq[i] = make_float4(aq[4 * i] / n, aq[4 * i + 1] / n, aq[4 * i + 2] / n, aq[4 * i + 3] / n);
                dk[i] = make_float4(ak[4 * i] / n, ak[4 * i + 1] / n, ak[4 * i + 2] / n, ak[4 * i + 3] / n);
            }
        }
    }
}

// ============================================================================ affinity + top-k

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

// One CTA per (image, block of `rows` = 8 NR rows), NR rows per warp. The image's key means and
// the block's query means (fp32 means, or the bf16 / fp32 tokens themselves when a region is one
// token) are staged in shared memory as fp32 a window of `chunk` channels at a time
// (the whole row when it fits), rows padded to chunk + 4 floats so that lanes reading different
// rows hit different banks; the partial sums carry over from window to window.
template <int E, bool ROUNDS, typename S>
__global__ void __launch_bounds__(256, 2) route_topk_kernel(const S *__restrict__ qm, const S *__restrict__ km,
                                                         int32_t *__restrict__ idx, int R, int C, int topk, int rows,
                                                         int chunk, float scale)
{
    extern __shared__ float4 smem4[];
    grid_dependency_wait();
    constexpr int NR = RowsPerPass<E>::value;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_blocks = (R + rows - 1) / rows;
    const int b = blockIdx.x / row_blocks;
    const int r0 = (blockIdx.x % row_blocks) * rows;
    const int nrows = min(rows, R - r0);
    const int stride = chunk + 4;
    const S *gkm = km + (int64_t)b * R * C;
    const S *gqm = qm + ((int64_t)b * R + r0) * C;
    float *skm = reinterpret_cast<float *>(smem4);
    float *sqm = skm + (size_t)R * stride;
    const int i0 = warp * NR;  // this warp's first row in the block
    const int nr = min(NR, nrows - i0);
    float acc[NR][E][4];
#pragma unroll
    for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int e = 0; e < E; ++e)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][e][j] = 0.f;
    for (int c0 = 0; c0 < C; c0 += chunk) {
        const int cn = min(chunk, C - c0);
        if (c0 > 0) __syncthreads();  // the previous window is no longer read
        stage_rows<false, S>(gkm, R, gqm, nrows, skm, C, c0, cn, stride);
        __syncthreads();
        if (nr > 0) affinity_accumulate<E, NR>(acc, sqm + (size_t)i0 * stride, stride, nr, skm, stride, R, cn, lane);
    }
    if (nr > 0) affinity_select<E, NR, ROUNDS>(acc, nr, R, topk, scale, idx + ((int64_t)b * R + r0 + i0) * topk, lane);
}

// Per-head routing ("医学图像分割模块", §五 steps ③④): the same rows, staging and selection as
// route_topk_kernel, for one head at a time: head h's means are channels [h hd, (h + 1) hd) of
// the region means (row stride C), its affinities are scaled by hd^-1/2, and its index rows go to
// idx[b, h, :, :]. One CTA per (image, head, block of rows); when a head's channels fit one
// staging pass, the block may hold more rows than its warps take at once, and the warps then
// go over them in turn on the same staged key means (fewer CTAs stage the same key rows).
template <int E, bool ROUNDS, typename S>
__global__ void __launch_bounds__(256, 2) route_heads_kernel(const S *__restrict__ qm, const S *__restrict__ km,
                                                          int32_t *__restrict__ idx, int R, int C, int hd, int heads,
                                                          int topk, int rows, int chunk, float scale)
{
    extern __shared__ float4 smem4[];
    grid_dependency_wait();
    constexpr int NR = RowsPerPass<E>::value;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_blocks = (R + rows - 1) / rows;
    const int bh = blockIdx.x / row_blocks;  // image * heads + head
    const int h = bh % heads, b = bh / heads;
    const int r0 = (blockIdx.x % row_blocks) * rows;
    const int nrows = min(rows, R - r0);
    const int stride = chunk + 4;
    const S *gkm = km + (int64_t)b * R * C + (int64_t)h * hd;
    const S *gqm = qm + ((int64_t)b * R + r0) * C + (int64_t)h * hd;
    float *skm = reinterpret_cast<float *>(smem4);
    float *sqm = skm + (size_t)R * stride;
    const int i0 = warp * NR;
    const int nr = min(NR, nrows - i0);
    float acc[NR][E][4];
    if (hd <= chunk) {
        stage_rows<false, S>(gkm, R, gqm, nrows, skm, C, 0, hd, stride);
        __syncthreads();
        for (int p0 = i0; p0 < nrows; p0 += 8 * NR) {  // 8 warps x NR rows per turn
            const int np = min(NR, nrows - p0);
#pragma unroll
            for (int i = 0; i < NR; ++i)
#pragma unroll
                for (int e = 0; e < E; ++e)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][e][j] = 0.f;
            affinity_accumulate<E, NR>(acc, sqm + (size_t)p0 * stride, stride, np, skm, stride, R, hd, lane);
            affinity_select<E, NR, ROUNDS>(acc, np, R, topk, scale, idx + ((int64_t)bh * R + r0 + p0) * topk, lane);
        }
        return;
    }
#pragma unroll
    for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int e = 0; e < E; ++e)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][e][j] = 0.f;
    for (int c0 = 0; c0 < hd; c0 += chunk) {
        const int cn = min(chunk, hd - c0);
        if (c0 > 0) __syncthreads();
        stage_rows<false, S>(gkm, R, gqm, nrows, skm, C, c0, cn, stride);
        __syncthreads();
        if (nr > 0) affinity_accumulate<E, NR>(acc, sqm + (size_t)i0 * stride, stride, nr, skm, stride, R, cn, lane);
    }
    if (nr > 0)
        affinity_select<E, NR, ROUNDS>(acc, nr, R, topk, scale, idx + ((int64_t)bh * R + r0 + i0) * topk, lane);
}

// Wide rows (R > 256): one warp per row, keys in shared memory, bitonic network there.
__global__ void __launch_bounds__(256) route_topk_wide_kernel(const float *__restrict__ qm,
                                                              const float *__restrict__ km, int32_t *__restrict__ idx,
                                                              int R, int C, int topk, int P, float scale)
{
    extern __shared__ unsigned long long keys[];
    grid_dependency_wait();
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

// ============================================================================ means kernels

// Means of rs > 16 regions: several regions per CTA.
template <typename T>
__global__ void __launch_bounds__(kMeansThreads, 2) region_means_kernel(const MeansArgs a)
{
    extern __shared__ float4 smem4[];
    grid_dependency_wait();
    const long long i0 = (long long)blockIdx.x * a.rpc;
    const int nreg = (int)min((long long)a.rpc, (long long)a.B * a.R - i0);
    region_means_block<T>(a, reinterpret_cast<float *>(smem4), i0, nreg);
}

// Means of rs <= 16 regions: one CTA per region, a multiple of 32 threads (every warp whole for
// the butterfly).
template <typename T>
__global__ void __launch_bounds__(256) region_means_small_kernel(const MeansArgs a, int lshift)
{
    grid_dependency_wait();
    region_means_small<T>(a, blockIdx.x / a.R, blockIdx.x % a.R, lshift);
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

// Regions per CTA of the means kernels: one group of `slots` threads (the region row segment's
// vectors, rounded up to a warp) per region, as many as fit in 256 threads.
static MeansArgs means_args(const void *q, const void *k, float *qm, float *km, const Geometry &g, bool bf16)
{
    MeansArgs a;
    a.q = q;
    a.k = k;
    a.qm = qm;
    a.km = km;
    a.B = g.B;
    a.H = g.H;
    a.W = g.W;
    a.C = g.C;
    a.n_win = g.n_win;
    a.hr = g.hr;
    a.wr = g.wr;
    a.R = g.R;
    const int V = bf16 ? 8 : 4;
    const int nvec = g.wr * (g.C / V);
    a.slots = nvec >= kMeansThreads ? kMeansThreads : (nvec + 31) / 32 * 32;
    a.rpc = kMeansThreads / a.slots;
    return a;
}

static size_t means_part_bytes(const MeansArgs &a) { return (size_t)a.rpc * 2 * a.wr * a.C * sizeof(float); }

static long long means_blocks(const MeansArgs &a) { return ((long long)a.B * a.R + a.rpc - 1) / a.rpc; }


cudaError_t launch_region_means(const void *q, const void *k, float *qm, float *km, const Geometry &g, bool bf16,
                                int num_sms, cudaStream_t stream)
{
    (void)num_sms;
    const MeansArgs a = means_args(q, k, qm, km, g, bf16);
    if ((long long)a.wr * (g.C / (bf16 ? 8 : 4)) > kMaxMeansVectors) return cudaErrorInvalidConfiguration;
    if ((long long)g.B * g.R > 0x7fffffffLL) return cudaErrorInvalidConfiguration;  // 32-bit region index
    if (g.rs <= 16) {
        const int lshift = g.hr == 8 ? 3 : (g.hr == 4 ? 2 : (g.hr == 2 ? 1 : 0));
        long long threads = ((long long)(g.C / (bf16 ? 8 : 4)) << lshift);
        threads = (threads + 31) / 32 * 32;
        if (threads > 256) threads = 256;
        const long long blocks = (long long)g.B * g.R;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        if (bf16)
            return launch_pdl(region_means_small_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3((unsigned)threads),
                              0, stream, a, lshift);
        return launch_pdl(region_means_small_kernel<float>, dim3((unsigned)blocks), dim3((unsigned)threads), 0, stream, a,
                          lshift);
    }
    const size_t smem = means_part_bytes(a);
    static int granted[2][64] = {{0}};
    cudaError_t e = bf16 ? raise_smem_limit(region_means_kernel<__nv_bfloat16>, smem, granted[0])
                         : raise_smem_limit(region_means_kernel<float>, smem, granted[1]);
    if (e != cudaSuccess) return e;
    const long long blocks = means_blocks(a);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (bf16)
        return launch_pdl(region_means_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(kMeansThreads), smem, stream,
                          a);
    return launch_pdl(region_means_kernel<float>, dim3((unsigned)blocks), dim3(kMeansThreads), smem, stream, a);
}

template <int E, bool ROUNDS, typename S>
static cudaError_t launch_topk_typed(const S *qm, const S *km, int32_t *idx, const Geometry &g, int rows, int chunk,
                                     float scale, size_t smem, cudaStream_t stream)
{
    static int granted[64] = {0};
    cudaError_t e = raise_smem_limit(route_topk_kernel<E, ROUNDS, S>, smem, granted);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)((g.R + rows - 1) / rows) * g.B;
    return launch_pdl(route_topk_kernel<E, ROUNDS, S>, dim3((unsigned)blocks), dim3(256), smem, stream, qm, km, idx, g.R,
                      g.C, g.topk, rows, chunk, scale);
}

template <int E, typename S>
static cudaError_t launch_topk_e(const S *qm, const S *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    const float scale = (float)(1.0 / sqrt((double)g.C));
    const bool rounds = topk_by_rounds(E, g.topk);
    // one pass of the row routine per warp: every warp of the CTA busy, the image's key means
    // staged once per channel window; the window is the whole row when the staged rows fit in
    // 100 KB, else the widest power-of-two multiple of 32 channels that does (a row stride of
    // 4 mod 32 words keeps the lanes' 16-byte key loads free of bank conflicts, and the window's
    // 16-byte vectors divide the CTA, which keeps the staging free of divisions)
    const int rows = 8 * RowsPerPass<E>::value;
    const long long per_col = (long long)(g.R + rows) * sizeof(float);
    int chunk = g.C;
    if (per_col * (chunk + 4) > 100 * 1024) {
        chunk = 32;
        while (chunk * 2 < g.C && per_col * (chunk * 2 + 4) <= 100 * 1024) chunk *= 2;
        if (per_col * (chunk + 4) > 100 * 1024) return cudaErrorInvalidConfiguration;  // R is at most 256 here
    }
    const size_t smem = (size_t)per_col * (chunk + 4);
    return rounds ? launch_topk_typed<E, true, S>(qm, km, idx, g, rows, chunk, scale, smem, stream)
                  : launch_topk_typed<E, false, S>(qm, km, idx, g, rows, chunk, scale, smem, stream);
}

static cudaError_t launch_route_tf32x3(const float *qm, const float *km, int32_t *idx, const Geometry &g,
                                       cudaStream_t stream);
// 3xTF32 routing for 64 < R <= 256 (E = 4 or 8 keys per lane in the selection): one CTA per
// (image, 16 query rows); the 8-key tiles are dealt to the warps (warp w takes tiles w, w + 8,
// w + 16, w + 24), and each warp forms whole dot products of its tiles over all channels, in
// 16-channel chunks with the same split, permutation and MMA order as route_tf32x3_kernel. The
// 16 x R tile goes to shared memory, then warp w selects the top-k of rows 2 w and 2 w + 1.
template <int E, bool ROUNDS>
__global__ void __launch_bounds__(256, 2) route_tf32x3_wide_kernel(const float *__restrict__ qm,
                                                                   const float *__restrict__ km,
                                                                   int32_t *__restrict__ idx, int R, int C, int topk,
                                                                   float scale)
{
    constexpr int kStride = 32 * E + 4;
    __shared__ float aff[16][kStride];
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int row_blocks = (R + 15) >> 4;
    const int b = blockIdx.x / row_blocks;
    const int r0 = (blockIdx.x - b * row_blocks) * 16;
    const int ntiles = (R + 7) >> 3;
    const float *qb = qm + (int64_t)b * R * C;
    const float *kb = km + (int64_t)b * R * C;
    const int ra = min(r0 + g, R - 1) * C + 4 * c, rb = min(r0 + g + 8, R - 1) * C + 4 * c;
    constexpr int T = E / 2;  // tiles per warp: 32 E / 8 keys over 8 warps
    int kr[T];
#pragma unroll
    for (int i = 0; i < T; ++i) kr[i] = min(8 * (warp + 8 * i) + g, R - 1) * C + 4 * c;
    float acc[T][4];
#pragma unroll
    for (int i = 0; i < T; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int col = 0; col < C; col += 16) {
        const float4 xa = __ldg(reinterpret_cast<const float4 *>(qb + ra + col));
        const float4 xb = __ldg(reinterpret_cast<const float4 *>(qb + rb + col));
        float4 y[T];
#pragma unroll
        for (int i = 0; i < T; ++i)
            if (warp + 8 * i < ntiles) y[i] = __ldg(reinterpret_cast<const float4 *>(kb + kr[i] + col));
        uint32_t ah[2][4], al[2][4];
        split_tf32(xa.x, ah[0][0], al[0][0]);
        split_tf32(xb.x, ah[0][1], al[0][1]);
        split_tf32(xa.y, ah[0][2], al[0][2]);
        split_tf32(xb.y, ah[0][3], al[0][3]);
        split_tf32(xa.z, ah[1][0], al[1][0]);
        split_tf32(xb.z, ah[1][1], al[1][1]);
        split_tf32(xa.w, ah[1][2], al[1][2]);
        split_tf32(xb.w, ah[1][3], al[1][3]);
#pragma unroll
        for (int i = 0; i < T; ++i)
            if (warp + 8 * i < ntiles) {
                uint32_t bh[4], bl[4];
                split_tf32(y[i].x, bh[0], bl[0]);
                split_tf32(y[i].y, bh[1], bl[1]);
                split_tf32(y[i].z, bh[2], bl[2]);
                split_tf32(y[i].w, bh[3], bl[3]);
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    mma_tf32_1688(acc[i], al[m], bh[2 * m], bh[2 * m + 1]);
                    mma_tf32_1688(acc[i], ah[m], bl[2 * m], bl[2 * m + 1]);
                    mma_tf32_1688(acc[i], ah[m], bh[2 * m], bh[2 * m + 1]);
                }
            }
    }
#pragma unroll
    for (int i = 0; i < T; ++i)
        if (warp + 8 * i < ntiles) {
            const int s0 = 8 * (warp + 8 * i) + 2 * c;
            *reinterpret_cast<float2 *>(&aff[g][s0]) = make_float2(acc[i][0], acc[i][1]);
            *reinterpret_cast<float2 *>(&aff[g + 8][s0]) = make_float2(acc[i][2], acc[i][3]);
        }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int rr = 2 * warp + i;
        if (r0 + rr >= R) break;
        unsigned long long key[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int s = 32 * e + lane;
            key[e] = s < R ? routing_key(aff[rr][s] * scale, s) : 0ull;
        }
        select_topk<E, ROUNDS>(key, topk, idx + ((int64_t)b * R + r0 + rr) * topk, lane);
    }
}

template <int E>
static cudaError_t launch_route_tf32x3_wide(const float *qm, const float *km, int32_t *idx, const Geometry &g,
                                            cudaStream_t stream)
{
    const long long blocks = (long long)g.B * ((g.R + 15) / 16);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const float scale = (float)(1.0 / sqrt((double)g.C));
    if (topk_by_rounds(E, g.topk))
        return launch_pdl(route_tf32x3_wide_kernel<E, true>, dim3((unsigned)blocks), dim3(256), 0, stream, qm, km, idx,
                          g.R, g.C, g.topk, scale);
    return launch_pdl(route_tf32x3_wide_kernel<E, false>, dim3((unsigned)blocks), dim3(256), 0, stream, qm, km, idx,
                      g.R, g.C, g.topk, scale);
}

bool route_tf32x3_supports(const Geometry &g);

template <typename S>
static cudaError_t launch_topk_any(const S *qm, const S *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    if constexpr (std::is_same<S, float>::value)
        if (route_tf32x3_supports(g)) return launch_route_tf32x3(qm, km, idx, g, stream);
    if (g.R <= 32) return launch_topk_e<1, S>(qm, km, idx, g, stream);
    if (g.R <= 64) return launch_topk_e<2, S>(qm, km, idx, g, stream);
    if (g.R <= 128) return launch_topk_e<4, S>(qm, km, idx, g, stream);
    return launch_topk_e<8, S>(qm, km, idx, g, stream);
}

// Tensor-core routing for up to 64 regions. One CTA per (image, 16 query rows); warp w takes
// channel chunks w, w + 8, ... and accumulates the 16 x 64 tile of partial dot products of its
// chunks with mma.sync, straight from 16-byte global loads, every load of the warp in flight at
// once. Within a chunk, lane (g, c) loads the same channel window of query rows g and g + 8 and
// of key g of each 8-key tile; the MMA's k slots take those channels in the same permuted order
// for A and B, which a sum over channels does not see. The eight partial tiles are then added
// in warp order in shared memory and warp w selects the top-k of rows 2 w and 2 w + 1 as every
// routing kernel does.
//  * bf16 one-token regions (route_tokens_mma_kernel): the means are the tokens, and a product
//    of two bf16 values is exact in fp32, so m16n8k16 bf16 MMAs with fp32 accumulation add the
//    same exact products an fp32 FMA path would, in another order (8 channels per lane). Here
//    warp w takes the 64-channel blocks w, w + 8, ..., each as its two 32-channel chunks in
//    order: with C <= 512 a warp's partial is exactly one block's, which is how the fused
//    route-and-attend kernel of the forward pass (one CTA per block) forms the same partials
//    and adds them in the same order, so both give the same index bits.
//  * fp32 means or tokens (route_tf32x3_kernel): each value is split into two tf32 parts,
//    x = hi + lo with |x - hi - lo| <= 2^-22 |x|, and m16n8k8 tf32 MMAs add lo*hi, hi*lo and
//    hi*hi (smallest first; lo*lo, below 2^-22 of the product, is left out). Every product is
//    exact in fp32, so an affinity is off by at most about 1e-6 of the sum of its terms'
//    magnitudes plus fp32 accumulation, and equal inputs give equal affinities (16-channel
//    chunks, 4 channels per lane).
constexpr int kRouteWarps = 8, kPartPad = 68;  // row stride of a partial tile (floats)

// acc[n][0..1]: row g, keys 8 n + 2 c, + 1; acc[n][2..3]: row g + 8, the same keys
__device__ __forceinline__ void store_partials(float (*part)[16][kPartPad], const float (&acc)[8][4], int ntiles,
                                               int warp, int g, int c)
{
#pragma unroll
    for (int n = 0; n < 8; ++n)
        if (n < ntiles) {
            *reinterpret_cast<float2 *>(&part[warp][g][8 * n + 2 * c]) = make_float2(acc[n][0], acc[n][1]);
            *reinterpret_cast<float2 *>(&part[warp][g + 8][8 * n + 2 * c]) = make_float2(acc[n][2], acc[n][3]);
        }
}

template <bool ROUNDS>
__device__ __forceinline__ void select_from_partials(float (*part)[16][kPartPad], int R, int r0, int ntiles,
                                                     int topk, float scale, int32_t *idx_image, int warp, int lane)
{
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int rr = 2 * warp + i;
        if (r0 + rr >= R) break;
        unsigned long long key[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int s = 32 * e + lane;
            float d = 0.f;
#pragma unroll
            for (int w = 0; w < kRouteWarps; ++w) d += (s < 8 * ntiles) ? part[w][rr][s] : 0.f;
            key[e] = s < R ? routing_key(d * scale, s) : 0ull;
        }
        select_topk<2, ROUNDS>(key, topk, idx_image + (int64_t)(r0 + rr) * topk, lane);
    }
}

template <bool ROUNDS>
__global__ void __launch_bounds__(256, 2) route_tokens_mma_kernel(const __nv_bfloat16 *__restrict__ q,
                                                                  const __nv_bfloat16 *__restrict__ k,
                                                                  int32_t *__restrict__ idx, int R, int C, int topk,
                                                                  float scale)
{
    __shared__ float part[kRouteWarps][16][kPartPad];
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int row_blocks = (R + 15) >> 4;
    const int b = blockIdx.x / row_blocks;
    const int r0 = (blockIdx.x - b * row_blocks) * 16;
    const int ntiles = (R + 7) >> 3;
    const __nv_bfloat16 *qb = q + (int64_t)b * R * C;
    const __nv_bfloat16 *kb = k + (int64_t)b * R * C;
    // offsets inside the image (R * C < 2^31, checked by the launcher); rows and keys past R
    // read row R - 1, and their results are never selected
    const int ra = min(r0 + g, R - 1) * C + 8 * c, rb = min(r0 + g + 8, R - 1) * C + 8 * c;
    int kr[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) kr[n] = min(8 * n + g, R - 1) * C + 8 * c;
    float acc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[n][j] = 0.f;
    for (int col = 64 * warp; col < C; col += (col & 32) ? 64 * kRouteWarps - 32 : 32) {
        const uint4 xa = __ldg(reinterpret_cast<const uint4 *>(qb + ra + col));
        const uint4 xb = __ldg(reinterpret_cast<const uint4 *>(qb + rb + col));
        uint4 y[8];
#pragma unroll
        for (int n = 0; n < 8; ++n)
            if (n < ntiles) y[n] = __ldg(reinterpret_cast<const uint4 *>(kb + kr[n] + col));
        const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};  // k slots 2c, 2c+1 | 2c+8, 2c+9: channels 8c..8c+3
        const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};  // channels 8c+4 .. 8c+7
#pragma unroll
        for (int n = 0; n < 8; ++n)
            if (n < ntiles) {
                mma_bf16_16816(acc[n], a0, y[n].x, y[n].y);
                mma_bf16_16816(acc[n], a1, y[n].z, y[n].w);
            }
    }
    store_partials(part, acc, ntiles, warp, g, c);
    __syncthreads();
    select_from_partials<ROUNDS>(part, R, r0, ntiles, topk, scale, idx + (int64_t)b * R * topk, warp, lane);
}

template <bool ROUNDS>
__global__ void __launch_bounds__(256, 2) route_tf32x3_kernel(const float *__restrict__ qm,
                                                              const float *__restrict__ km,
                                                              int32_t *__restrict__ idx, int R, int C, int topk,
                                                              float scale)
{
    __shared__ float part[kRouteWarps][16][kPartPad];
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int row_blocks = (R + 15) >> 4;
    const int b = blockIdx.x / row_blocks;
    const int r0 = (blockIdx.x - b * row_blocks) * 16;
    const int ntiles = (R + 7) >> 3;
    const float *qb = qm + (int64_t)b * R * C;
    const float *kb = km + (int64_t)b * R * C;
    const int ra = min(r0 + g, R - 1) * C + 4 * c, rb = min(r0 + g + 8, R - 1) * C + 4 * c;
    int kr[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) kr[n] = min(8 * n + g, R - 1) * C + 4 * c;
    float acc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[n][j] = 0.f;
    for (int col = 16 * warp; col < C; col += 16 * kRouteWarps) {
        const float4 xa = __ldg(reinterpret_cast<const float4 *>(qb + ra + col));
        const float4 xb = __ldg(reinterpret_cast<const float4 *>(qb + rb + col));
        float4 y[8];
#pragma unroll
        for (int n = 0; n < 8; ++n)
            if (n < ntiles) y[n] = __ldg(reinterpret_cast<const float4 *>(kb + kr[n] + col));
        // MMA m of the chunk: k slot c <- channel 4c + 2m, k slot c + 4 <- channel 4c + 2m + 1
        uint32_t ah[2][4], al[2][4];
        split_tf32(xa.x, ah[0][0], al[0][0]);
        split_tf32(xb.x, ah[0][1], al[0][1]);
        split_tf32(xa.y, ah[0][2], al[0][2]);
        split_tf32(xb.y, ah[0][3], al[0][3]);
        split_tf32(xa.z, ah[1][0], al[1][0]);
        split_tf32(xb.z, ah[1][1], al[1][1]);
        split_tf32(xa.w, ah[1][2], al[1][2]);
        split_tf32(xb.w, ah[1][3], al[1][3]);
#pragma unroll
        for (int n = 0; n < 8; ++n)
            if (n < ntiles) {
                uint32_t bh[4], bl[4];
                split_tf32(y[n].x, bh[0], bl[0]);
                split_tf32(y[n].y, bh[1], bl[1]);
                split_tf32(y[n].z, bh[2], bl[2]);
                split_tf32(y[n].w, bh[3], bl[3]);
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    mma_tf32_1688(acc[n], al[m], bh[2 * m], bh[2 * m + 1]);
                    mma_tf32_1688(acc[n], ah[m], bl[2 * m], bl[2 * m + 1]);
                    mma_tf32_1688(acc[n], ah[m], bh[2 * m], bh[2 * m + 1]);
                }
            }
    }
    store_partials(part, acc, ntiles, warp, g, c);
    __syncthreads();
    select_from_partials<ROUNDS>(part, R, r0, ntiles, topk, scale, idx + (int64_t)b * R * topk, warp, lane);
}

bool route_tf32x3_supports(const Geometry &g)
{
    return g.R <= 256 && g.C % 16 == 0 && (long long)g.R * g.C < (1LL << 31);
}

static cudaError_t launch_route_tf32x3(const float *qm, const float *km, int32_t *idx, const Geometry &g,
                                       cudaStream_t stream)
{
    const long long blocks = (long long)g.B * ((g.R + 15) / 16);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (g.R > 128) return launch_route_tf32x3_wide<8>(qm, km, idx, g, stream);
    if (g.R > 64) return launch_route_tf32x3_wide<4>(qm, km, idx, g, stream);
    const float scale = (float)(1.0 / sqrt((double)g.C));
    if (topk_by_rounds(2, g.topk))
        return launch_pdl(route_tf32x3_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, stream, qm, km, idx, g.R,
                          g.C, g.topk, scale);
    return launch_pdl(route_tf32x3_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, stream, qm, km, idx, g.R, g.C,
                      g.topk, scale);
}

bool route_tokens_mma_supports(const Geometry &g, bool bf16)
{
    return bf16 && g.rs == 1 && g.R <= 64 && g.C % 32 == 0 && (long long)g.R * g.C < (1LL << 31);
}

static cudaError_t launch_route_tokens_mma(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int32_t *idx,
                                           const Geometry &g, cudaStream_t stream)
{
    const long long blocks = (long long)g.B * ((g.R + 15) / 16);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const float scale = (float)(1.0 / sqrt((double)g.C));
    if (topk_by_rounds(2, g.topk))
        return launch_pdl(route_tokens_mma_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, stream, q, k, idx, g.R,
                          g.C, g.topk, scale);
    return launch_pdl(route_tokens_mma_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, stream, q, k, idx, g.R,
                      g.C, g.topk, scale);
}

cudaError_t launch_route_topk_tokens(const void *q, const void *k, int32_t *idx, const Geometry &g, bool bf16,
                                     cudaStream_t stream)
{
    if (g.rs != 1 || g.R > 256) return cudaErrorInvalidConfiguration;
    if (route_tokens_mma_supports(g, bf16))
        return launch_route_tokens_mma(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), idx,
                                       g, stream);
    return bf16 ? launch_topk_any<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(q),
                                                 static_cast<const __nv_bfloat16 *>(k), idx, g, stream)
                : launch_topk_any<float>(static_cast<const float *>(q), static_cast<const float *>(k), idx, g, stream);
}

cudaError_t launch_route_topk(const float *qm, const float *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    if (g.R <= 256) return launch_topk_any<float>(qm, km, idx, g, stream);
    int P = 512;
    while (P < g.R) P <<= 1;
    int warps = (int)((48 * 1024) / ((size_t)P * 8));
    if (warps > 8) warps = 8;
    const long long blocks = (long long)((g.R + warps - 1) / warps) * g.B;
    const float scale = (float)(1.0 / sqrt((double)g.C));
    return launch_pdl(route_topk_wide_kernel, dim3((unsigned)blocks), dim3(warps * 32), (size_t)warps * P * 8, stream, qm,
                      km, idx, g.R, g.C, g.topk, P, scale);
}

}  // namespace bra

namespace bra {

template <int E, bool ROUNDS, typename S>
static cudaError_t launch_heads_typed(const S *qm, const S *km, int32_t *idx, const Geometry &g, int rows, int chunk,
                                      float scale, size_t smem, cudaStream_t stream)
{
    static int granted[64] = {0};
    cudaError_t e = raise_smem_limit(route_heads_kernel<E, ROUNDS, S>, smem, granted);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)((g.R + rows - 1) / rows) * g.B * g.heads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return launch_pdl(route_heads_kernel<E, ROUNDS, S>, dim3((unsigned)blocks), dim3(256), smem, stream, qm, km, idx,
                      g.R, g.C, g.hd, g.heads, g.topk, rows, chunk, scale);
}

template <int E, typename S>
static cudaError_t launch_heads_e(const S *qm, const S *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    const float scale = (float)(1.0 / sqrt((double)g.hd));
    const int turn = 8 * RowsPerPass<E>::value;  // rows the warps take at once
    int rows = turn;
    // one staging pass for the whole head: blocks of several turns of rows, about two CTAs per SM
    // in all (the key means of an (image, head) are then staged by fewer CTAs)
    {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const long long pairs = (long long)g.B * g.heads;
        long long blocks_per_pair = (2LL * sms + pairs - 1) / pairs;
        if (blocks_per_pair < 1) blocks_per_pair = 1;
        int want = (int)((g.R + blocks_per_pair - 1) / blocks_per_pair);
        want = (want + turn - 1) / turn * turn;
        if ((long long)(g.R + want) * sizeof(float) * (g.hd + 4) <= 100 * 1024 && want > rows) rows = want;
    }
    long long per_col = (long long)(g.R + rows) * sizeof(float);
    constexpr int V = 16 / sizeof(S);
    int chunk = g.hd;
    if (per_col * (chunk + 4) > 100 * 1024) {
        rows = turn;  // several staging passes: one turn of rows per CTA
        per_col = (long long)(g.R + rows) * sizeof(float);
        chunk = 32;
        while (chunk * 2 < g.hd && per_col * (chunk * 2 + 4) <= 100 * 1024) chunk *= 2;
        if (per_col * (chunk + 4) > 100 * 1024) return cudaErrorInvalidConfiguration;
    }
    if (chunk % V != 0) return cudaErrorInvalidConfiguration;
    const size_t smem = (size_t)per_col * (chunk + 4);
    return topk_by_rounds(E, g.topk) ? launch_heads_typed<E, true, S>(qm, km, idx, g, rows, chunk, scale, smem, stream)
                                     : launch_heads_typed<E, false, S>(qm, km, idx, g, rows, chunk, scale, smem, stream);
}

template <typename S>
static cudaError_t launch_heads_any(const S *qm, const S *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    if (g.R <= 32) return launch_heads_e<1, S>(qm, km, idx, g, stream);
    if (g.R <= 64) return launch_heads_e<2, S>(qm, km, idx, g, stream);
    if (g.R <= 128) return launch_heads_e<4, S>(qm, km, idx, g, stream);
    if (g.R <= 256) return launch_heads_e<8, S>(qm, km, idx, g, stream);
    return cudaErrorInvalidConfiguration;
}

bool route_heads_supports(const Geometry &g, bool bf16)
{
    // each head's slice of a row starts on a 16-byte boundary: of the fp32 means, and of the
    // tokens themselves when a region is one token
    const int elem = (g.rs == 1) ? (bf16 ? 2 : 4) : 4;
    return g.R <= 256 && (g.hd * elem) % 16 == 0 && (g.hd * 4) % 16 == 0;
}

cudaError_t launch_route_heads(const float *qm, const float *km, int32_t *idx, const Geometry &g, cudaStream_t stream)
{
    return launch_heads_any<float>(qm, km, idx, g, stream);
}

cudaError_t launch_route_heads_tokens(const void *q, const void *k, int32_t *idx, const Geometry &g, bool bf16,
                                      cudaStream_t stream)
{
    if (g.rs != 1) return cudaErrorInvalidConfiguration;
    return bf16 ? launch_heads_any<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(q),
                                                  static_cast<const __nv_bfloat16 *>(k), idx, g, stream)
                : launch_heads_any<float>(static_cast<const float *>(q), static_cast<const float *>(k), idx, g, stream);
}

}  // namespace bra

namespace bra {

// Region means of a padded map (auto_pad, "从静态到动态", §4.2): the region grid covers
// n_win hr x n_win wr tokens, of which those at y >= H or x >= W lie outside the H x W image and
// are zeros. One warp per region; lane l sums the channel vectors l, l + 32, ... over the
// region's tokens inside the image in row-major order (four tokens' loads in flight), and the sum
// is divided by hr wr (the zeros count).
template <typename T>
__global__ void __launch_bounds__(256) region_means_padded_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                                  float *__restrict__ qm, float *__restrict__ km,
                                                                  int B, int H, int W, int C, int n_win, int hr,
                                                                  int wr)
{
    grid_dependency_wait();
    constexpr int V = Vec16<T>::N;
    const int R = n_win * n_win;
    const long long reg = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (reg >= (long long)B * R) return;
    const int lane = threadIdx.x & 31;
    const long long b = reg / R;
    const int r = (int)(reg - b * R);
    const int ry = r / n_win, rx = r - ry * n_win;
    const int y1 = min(H, (ry + 1) * hr), x1 = min(W, (rx + 1) * wr);
    const float n = (float)(hr * wr);
    const int x0 = rx * wr, nx = x1 - x0, y0 = ry * hr;
    const int ntok = (y1 - y0) * nx;  // the region's tokens inside the image, row-major
    constexpr int kBatch = 4;         // tokens' loads of q and of k in flight per lane
    for (int v = lane; v < C / V; v += 32) {
        float aq[V], ak[V];
#pragma unroll
        for (int i = 0; i < V; ++i) aq[i] = ak[i] = 0.f;
        for (int t0 = 0; t0 < ntok; t0 += kBatch) {
            uint4 rq[kBatch], rk[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                if (t0 + u < ntok) {
                    const int t = t0 + u, y = y0 + t / nx, x = x0 + t % nx;
                    const int64_t off = ((b * H + y) * W + x) * C + (int64_t)v * V;
                    rq[u] = Vec16<T>::load_raw(q + off);
                    rk[u] = Vec16<T>::load_raw(k + off);
                }
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                if (t0 + u < ntok) {
                    Vec16<T>::accumulate(rq[u], aq);
                    Vec16<T>::accumulate(rk[u], ak);
                }
        }
        float4 *dq = reinterpret_cast<float4 *>(qm + reg * C + (int64_t)v * V);
        float4 *dk = reinterpret_cast<float4 *>(km + reg * C + (int64_t)v * V);
#pragma unroll
        for (int i = 0; i < V / 4; ++i) {
            dq[i] = make_float4(aq[4 * i] / n, aq[4 * i + 1] / n, aq[4 * i + 2] / n, aq[4 * i + 3] / n);
            dk[i] = make_float4(ak[4 * i] / n, ak[4 * i + 1] / n, ak[4 * i + 2] / n, ak[4 * i + 3] / n);
        }
    }
}

cudaError_t launch_region_means_padded(const void *q, const void *k, float *qm, float *km, const Geometry &g, int H,
                                       int W, bool bf16, cudaStream_t stream)
{
    const long long blocks = ((long long)g.B * g.R + 7) / 8;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (bf16)
        return launch_pdl(region_means_padded_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(256), 0, stream,
                          static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), qm, km, g.B, H,
                          W, g.C, g.n_win, g.hr, g.wr);
    return launch_pdl(region_means_padded_kernel<float>, dim3((unsigned)blocks), dim3(256), 0, stream,
                      static_cast<const float *>(q), static_cast<const float *>(k), qm, km, g.B, H, W, g.C, g.n_win,
                      g.hr, g.wr);
}

}  // namespace bra
