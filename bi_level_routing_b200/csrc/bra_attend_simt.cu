// bra_attend_simt.cu -- token-to-token attention over the routed regions on CUDA cores.
//
// For every query token of region r and every head: softmax, scale head_dim^-1/2, over the
// tokens of the routed regions (in idx order, row-major inside a region), then the weighted sum
// of their values ("从零构建BiFormer", §2.2 TokenAttention; "医学图像分割模块：BiFormer / 双层路由
// 注意力", §五 steps ⑤-⑦). This is the kernel of every shape the tensor-core kernels do not take:
// fp32 inputs, head sizes other than 32, per-head routing (each head gathers the regions of its
// own index row, §五 steps ③④) and padded maps (auto_pad: tokens outside the H x W image are
// zeros, as keys and values; queries there are not computed).
//
// One CTA per (image, query region, group of heads): the routed regions' key and value rows of
// those heads are staged in shared memory by the whole CTA (16-byte vectors when a head's
// channels allow it), a chunk of routed regions at a time; then `ks` threads per (query token,
// head) (consecutive lanes; ks = 1 when the queries and heads of a CTA fill 256 threads, up to 8
// for small regions) each keep q and a partial output in registers and fold the softmax online
// over every ks-th staged key (running max and sum, exp2 with a log2(e) pre-scale); the ks
// partial states are merged by warp shuffles at the end. The gathered K/V never reach HBM.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

struct StagedArgs {
    const void *q, *k, *v;
    const int32_t *idx;
    void *out;
    unsigned *err;
    int H, W;  // the image; the region grid may cover more (tokens outside are zeros)
    int C, heads, hd, n_win, hr, wr, rs, R, topk;
    int per_head;  // idx is [B, heads, R, topk]; else [B, R, topk], shared by all heads
    int hpc;       // heads per CTA
    int tq;        // query tokens per head and pass
    int ks;        // threads per (query token, head): the keys are dealt among them
    int kchunk;    // routed regions staged per chunk
    int vec;       // head rows staged as 16-byte vectors
    float scale_log2;
};

}  // namespace

template <typename T, int HDMAX>
__global__ void __launch_bounds__(256) attend_staged_kernel(const StagedArgs a)
{
    extern __shared__ float4 smem4[];
    const int ngroups = a.heads / a.hpc;
    int64_t blk = blockIdx.x;
    const int hg = (int)(blk % ngroups);
    blk /= ngroups;
    const int r = (int)(blk % a.R);
    const int64_t b = blk / a.R;
    const int ry = r / a.n_win, rx = r - ry * a.n_win;
    const int nkc = a.kchunk * a.rs;  // staged keys per head and chunk
    // a head's rows start 16 bytes past a multiple of 128: heads that share a warp (regions of
    // fewer than 32 tokens) read their rows from different banks
    const size_t hstride = (size_t)nkc * a.hd + 16 / sizeof(T);
    T *Ks = reinterpret_cast<T *>(smem4);              // [hpc] x hstride: [nkc][hd]
    T *Vs = Ks + (size_t)a.hpc * hstride;              // [hpc] x hstride: [nkc][hd]
    int *sreg = reinterpret_cast<int *>((reinterpret_cast<uintptr_t>(Vs + (size_t)a.hpc * hstride) + 15) &
                                        ~uintptr_t(15));  // [hpc][kchunk]: region, or -1
    const T *gq = static_cast<const T *>(a.q);
    const T *gk = static_cast<const T *>(a.k);
    const T *gv = static_cast<const T *>(a.v);
    T *gout = static_cast<T *>(a.out);
    const int qt = threadIdx.x / a.ks, kq = threadIdx.x - qt * a.ks;  // (head, query) slot; key lane
    const int hl = qt / a.tq, tt = qt - hl * a.tq;
    const int h = hg * a.hpc + hl;
    grid_dependency_wait();

    for (int t0 = 0; t0 < a.rs; t0 += a.tq) {  // passes over the region's query tokens
        const int t = t0 + tt;
        const int qy = ry * a.hr + (t < a.rs ? t / a.wr : 0), qx = rx * a.wr + (t < a.rs ? t % a.wr : 0);
        const bool real = hl < a.hpc && t < a.rs && qy < a.H && qx < a.W;
        const int64_t qoff = ((b * a.H + qy) * a.W + qx) * a.C + (int64_t)h * a.hd;
        float qv[HDMAX], o[HDMAX];
#pragma unroll
        for (int c = 0; c < HDMAX; ++c) {
            qv[c] = (real && c < a.hd) ? to_float(gq[qoff + c]) : 0.f;
            o[c] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        for (int j0 = 0; j0 < a.topk; j0 += a.kchunk) {
            const int nj = min(a.kchunk, a.topk - j0);
            __syncthreads();  // the previous chunk is no longer read
            for (int e = threadIdx.x; e < a.hpc * nj; e += blockDim.x) {
                const int ehl = e / nj, jj = e - ehl * nj;
                const int64_t row = a.per_head ? ((b * a.heads + hg * a.hpc + ehl) * a.R + r) : (b * a.R + r);
                const int s = a.idx[row * a.topk + j0 + jj];
                const bool ok = s >= 0 && s < a.R;
                if (!ok && t0 == 0) flag_error(a.err, kErrIndex);
                sreg[ehl * a.kchunk + jj] = ok ? s : -1;
            }
            __syncthreads();
            // stage the key and value rows (head, routed slot, token) of this chunk: 16-byte vectors,
            // four of k and four of v per thread in flight before their shared-memory stores
            const int rows = a.hpc * nj * a.rs;
            if (a.vec) {
                constexpr int kBatch = 4;
                const int per_row = (a.hd * (int)sizeof(T)) / 16, total = rows * per_row;
                for (int e0 = threadIdx.x; e0 < total; e0 += kBatch * blockDim.x) {
                    uint4 kv[kBatch], vv[kBatch];
                    size_t so[kBatch];
#pragma unroll
                    for (int i = 0; i < kBatch; ++i) {
                        const int e = e0 + i * blockDim.x;
                        kv[i] = vv[i] = make_uint4(0u, 0u, 0u, 0u);
                        so[i] = ~size_t(0);
                        if (e >= total) continue;
                        const int row = e / per_row, u = e - row * per_row;
                        const int ehl = row / (nj * a.rs), rem = row - ehl * (nj * a.rs);
                        const int jj = rem / a.rs, tk = rem - jj * a.rs;
                        const int s = sreg[ehl * a.kchunk + jj];
                        if (s < 0) continue;
                        so[i] = ehl * hstride + (size_t)(jj * a.rs + tk) * a.hd;
                        const int sy = s / a.n_win, sx = s - sy * a.n_win;
                        const int ky = sy * a.hr + tk / a.wr, kx = sx * a.wr + tk % a.wr;
                        so[i] += (size_t)u * (16 / sizeof(T));
                        if (ky < a.H && kx < a.W) {
                            const int64_t goff = ((b * a.H + ky) * a.W + kx) * a.C +
                                                 (int64_t)(hg * a.hpc + ehl) * a.hd + u * (16 / (int)sizeof(T));
                            kv[i] = __ldg(reinterpret_cast<const uint4 *>(gk + goff));
                            vv[i] = __ldg(reinterpret_cast<const uint4 *>(gv + goff));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < kBatch; ++i)
                        if (so[i] != ~size_t(0)) {
                            *reinterpret_cast<uint4 *>(Ks + so[i]) = kv[i];
                            *reinterpret_cast<uint4 *>(Vs + so[i]) = vv[i];
                        }
                }
            } else {
                for (int e = threadIdx.x; e < rows * a.hd; e += blockDim.x) {
                    const int row = e / a.hd, u = e - row * a.hd;
                    const int ehl = row / (nj * a.rs), rem = row - ehl * (nj * a.rs);
                    const int jj = rem / a.rs, tk = rem - jj * a.rs;
                    const int s = sreg[ehl * a.kchunk + jj];
                    if (s < 0) continue;
                    const int sy = s / a.n_win, sx = s - sy * a.n_win;
                    const int ky = sy * a.hr + tk / a.wr, kx = sx * a.wr + tk % a.wr;
                    const bool inside = ky < a.H && kx < a.W;
                    const int64_t goff = ((b * a.H + ky) * a.W + kx) * a.C + (int64_t)(hg * a.hpc + ehl) * a.hd;
                    const size_t soff = ehl * hstride + (size_t)(jj * a.rs + tk) * a.hd;
                    Ks[soff + u] = inside ? gk[goff + u] : from_float<T>(0.f);
                    Vs[soff + u] = inside ? gv[goff + u] : from_float<T>(0.f);
                }
            }
            __syncthreads();
            if (!real) continue;
            const T *kh = Ks + hl * hstride;
            const T *vh = Vs + hl * hstride;
            constexpr int V = Vec16<T>::N;
            for (int key = kq; key < nj * a.rs; key += a.ks) {  // this thread's keys of the chunk
                const int jj = key / a.rs;
                if (sreg[hl * a.kchunk + jj] < 0) continue;  // a skipped region contributes no key
                {
                    const T *kr = kh + (size_t)key * a.hd;
                    const T *vr = vh + (size_t)key * a.hd;
                    float dot = 0.f;
                    if (a.vec) {  // 16-byte rows: V channels per shared-memory load
#pragma unroll
                        for (int c0 = 0; c0 < HDMAX; c0 += V)
                            if (c0 < a.hd) {
                                float f[V];
                                Vec16<T>::load_shared(kr + c0, f);
#pragma unroll
                                for (int i = 0; i < V; ++i) dot = fmaf(qv[c0 + i], f[i], dot);
                            }
                    } else {
#pragma unroll
                        for (int c = 0; c < HDMAX; ++c)
                            if (c < a.hd) dot = fmaf(qv[c], to_float(kr[c]), dot);
                    }
                    const float sl = dot * a.scale_log2;  // logit in log2 units
                    if (sl > m) {
                        const float corr = fast_exp2(m - sl);
                        l *= corr;
#pragma unroll
                        for (int c = 0; c < HDMAX; ++c) o[c] *= corr;
                        m = sl;
                    }
                    const float p = fast_exp2(sl - m);
                    l += p;
                    if (a.vec) {
#pragma unroll
                        for (int c0 = 0; c0 < HDMAX; c0 += V)
                            if (c0 < a.hd) {
                                float f[V];
                                Vec16<T>::load_shared(vr + c0, f);
#pragma unroll
                                for (int i = 0; i < V; ++i) o[c0 + i] = fmaf(p, f[i], o[c0 + i]);
                            }
                    } else {
#pragma unroll
                        for (int c = 0; c < HDMAX; ++c)
                            if (c < a.hd) o[c] = fmaf(p, to_float(vr[c]), o[c]);
                    }
                }
            }
        }
        // merge the ks partial states of a (query, head): rescale to the common max, then add
        // (every lane of the warp takes part; lanes without a query hold m = -inf, l = 0)
        for (int off = 1; off < a.ks; off <<= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m, off);
            const float mn = fmaxf(m, mo);
            const float sc = (m == -INFINITY) ? 0.f : fast_exp2(m - mn);
            const float so = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mn);
            l = l * sc + __shfl_xor_sync(0xffffffffu, l, off) * so;
#pragma unroll
            for (int c = 0; c < HDMAX; ++c) o[c] = o[c] * sc + __shfl_xor_sync(0xffffffffu, o[c], off) * so;
            m = mn;
        }
        if (real && kq == 0) {
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < HDMAX; ++c)
                if (c < a.hd) gout[qoff + c] = from_float<T>(o[c] * inv);
        }
    }
}

namespace {

constexpr size_t kStagedMaxSmem = 96 * 1024;     // one routed region per chunk must fit
constexpr size_t kStagedTargetSmem = 32 * 1024;  // more regions per chunk while within this

template <typename T>
cudaError_t launch_staged_typed(StagedArgs a, const Geometry &g, cudaStream_t stream)
{
    const int elem = (int)sizeof(T);
    // heads per CTA: the largest divisor of heads with hpc * rs <= 256 threads
    int hpc = 1;
    for (int d = 1; d <= g.heads; ++d)
        if (g.heads % d == 0 && (long long)d * g.rs <= 256) hpc = d;
    a.hpc = hpc;
    a.tq = g.rs <= 256 ? g.rs : 256;
    // threads per (query, head): up to 8 while the CTA stays within 256 threads
    int ks = 1;
    while (ks < 8 && (long long)hpc * a.tq * ks * 2 <= 256) ks *= 2;
    a.ks = ks;
    int threads = ((hpc * a.tq * ks + 31) / 32) * 32;
    if (threads > 256) threads = 256;
    a.vec = ((g.hd * elem) % 16 == 0) ? 1 : 0;
    // routed regions per chunk: as many as keep the CTA within kStagedTargetSmem (several CTAs per
    // SM), at least one
    const size_t per_region = (size_t)2 * hpc * g.rs * g.hd * elem + 4 * (size_t)hpc;
    const size_t fixed = (size_t)2 * hpc * 16 + 32;  // the heads' 16-byte offsets, alignment slack
    if (per_region + fixed > kStagedMaxSmem) return cudaErrorInvalidConfiguration;
    long long kc = (long long)((kStagedTargetSmem - fixed) / per_region);
    if (kc < 1) kc = 1;
    if (kc > g.topk) kc = g.topk;
    a.kchunk = (int)kc;
    const size_t smem = (size_t)a.kchunk * per_region + fixed;
    const long long blocks = (long long)g.B * g.R * (g.heads / hpc);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    void (*kernel)(const StagedArgs) = g.hd <= 32 ? attend_staged_kernel<T, 32>
                                                  : (g.hd <= 64 ? attend_staged_kernel<T, 64> : attend_staged_kernel<T, 128>);
    static int granted[3][64] = {{0}};
    const int slot = g.hd <= 32 ? 0 : (g.hd <= 64 ? 1 : 2);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)smem > granted[slot][dev] && smem > 48 * 1024) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        granted[slot][dev] = (int)smem;
    }
    return launch_pdl(kernel, dim3((unsigned)blocks), dim3(threads), smem, stream, a);
}

}  // namespace

cudaError_t launch_attend_staged(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                                 const Geometry &g, int H, int W, bool per_head, bool bf16, unsigned *err,
                                 cudaStream_t stream)
{
    if (g.hd > kSimtMaxHeadDim) return cudaErrorInvalidConfiguration;
    StagedArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.idx = idx;
    a.out = out;
    a.err = err;
    a.H = H;
    a.W = W;
    a.C = g.C;
    a.heads = g.heads;
    a.hd = g.hd;
    a.n_win = g.n_win;
    a.hr = g.hr;
    a.wr = g.wr;
    a.rs = g.rs;
    a.R = g.R;
    a.topk = g.topk;
    a.per_head = per_head ? 1 : 0;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    return bf16 ? launch_staged_typed<__nv_bfloat16>(a, g, stream) : launch_staged_typed<float>(a, g, stream);
}

cudaError_t launch_attend_simt(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                               const Geometry &g, bool bf16, unsigned *err, cudaStream_t stream)
{
    return launch_attend_staged(q, k, v, idx, out, g, g.H, g.W, false, bf16, err, stream);
}

}  // namespace bra
