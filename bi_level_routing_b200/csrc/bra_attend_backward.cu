// bra_attend_backward.cu -- the backward pass of the token attention with the routing index held
// fixed: given dout = dL/dout, the gradients dq, dk, dv of L = sum(dout * out). The pages train
// the model ("从静态到动态", §3.2; "BiFormer用双层路由注意力重塑视觉Transformer效率极限", §3.2) but
// print no backward; top-k passes no gradient, so routing is a constant of the backward. Per
// query token and head, with logits l_i = hd^-1/2 q . k_i over the gathered keys and p = softmax:
//   dv_i += p_i dout,  dp_i = dout . v_i,  ds_i = p_i (dp_i - D),  D = sum_j p_j dp_j = dout . out,
//   dq = hd^-1/2 sum_i ds_i k_i,  dk_i += hd^-1/2 ds_i q.
//
// One CTA per (image, query region, group of heads), one thread per (query token, head):
//  pass 1 recomputes the forward softmax (running max and sum) over the staged keys and, with
//         the same rescaling, D = dout . out = sum_i p_i (dout . v_i);
//  pass 2 forms p_i and ds_i chunk by chunk, adds dq in registers (a query's keys are all in its
//         CTA, so dq is written once, without atomics), and keeps p and ds of the chunk in
//         shared memory; the CTA then turns around, one thread per (key, 4 channels), and sums
//         dk and dv of the chunk's keys over the region's queries, which it adds to global
//         memory with 16-byte atomics (other query regions route to the same keys).
// dq, dk, dv are fp32 [B, H, W, C] whatever the input type; dk and dv are cleared first.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

struct BackArgs {
    const void *q, *k, *v, *dout;
    const int32_t *idx;
    float *dq, *dk, *dv;
    unsigned *err;
    int H, W, C, heads, hd, n_win, hr, wr, rs, R, topk;
    int hpc;     // heads per CTA
    int kcr;     // routed regions per key chunk
    int nitems;  // (image, region, head) items of the persistent tensor-core kernel
    float scale;       // hd^-1/2
    float scale_log2;  // hd^-1/2 log2(e)
};

}  // namespace

// Copies one head row of `hd` elements of T (16-byte aligned, hd * sizeof(T) a multiple of 16) to
// fp32 in shared memory, one 16-byte vector per call: vector u of the row.
template <typename T>
__device__ __forceinline__ void row_vec_to_f32(float *dst, const T *src, int u)
{
    constexpr int V = Vec16<T>::N;
    float f[V];
    Vec16<T>::load(src + u * V, f);
    float4 *d = reinterpret_cast<float4 *>(dst + u * V);
#pragma unroll
    for (int i = 0; i < V / 4; ++i) d[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
}

template <typename T, int HDMAX>
__global__ void __launch_bounds__(256) attend_backward_kernel(const BackArgs a)
{
    extern __shared__ float4 smem4[];
    const int ngroups = a.heads / a.hpc;
    int64_t blk = blockIdx.x;
    const int hg = (int)(blk % ngroups);
    blk /= ngroups;
    const int r = (int)(blk % a.R);
    const int64_t b = blk / a.R;
    const int ry = r / a.n_win, rx = r - ry * a.n_win;
    const int hd = a.hd, rs = a.rs, hpc = a.hpc;
    const int kc = a.kcr * rs;  // keys per chunk and head
    // a head's staged key rows start 4 floats past a multiple of 32: the heads that share a warp
    // (regions of fewer than 32 tokens) read their rows from different banks
    const size_t hstride = (size_t)kc * hd + 4;
    float *Qs = reinterpret_cast<float *>(smem4);      // [hpc][rs][hd]
    float *Ds = Qs + (size_t)hpc * rs * hd;            // [hpc][rs][hd] dout
    float *Ks = Ds + (size_t)hpc * rs * hd;            // [hpc] x hstride: [kc][hd]
    float *Vs = Ks + (size_t)hpc * hstride;            // [hpc] x hstride: [kc][hd]
    float *Ps = Vs + (size_t)hpc * hstride;            // [hpc][kc][rs]: p of (key, query)
    float *Ss = Ps + (size_t)hpc * kc * rs;            // [hpc][kc][rs]: ds of (key, query)
    int *sreg = reinterpret_cast<int *>(Ss + (size_t)hpc * kc * rs);  // [hpc][topk]
    const T *gq = static_cast<const T *>(a.q), *gk = static_cast<const T *>(a.k);
    const T *gv = static_cast<const T *>(a.v), *gd = static_cast<const T *>(a.dout);
    const int hl = threadIdx.x / rs, t = threadIdx.x - hl * rs;
    const bool active = hl < hpc;
    const int h = hg * hpc + hl;
    const int nvh = hd / Vec16<T>::N;  // 16-byte vectors per head row
    grid_dependency_wait();

    // the region's queries and output gradients, and the routed regions of every head
    for (int e = threadIdx.x; e < hpc * rs * nvh; e += blockDim.x) {
        const int row = e / nvh, u = e - row * nvh;
        const int eh = row / rs, et = row - eh * rs;
        const int y = ry * a.hr + et / a.wr, x = rx * a.wr + et % a.wr;
        const int64_t off = ((b * a.H + y) * a.W + x) * a.C + (int64_t)(hg * hpc + eh) * hd;
        row_vec_to_f32(Qs + (size_t)row * hd, gq + off, u);
        row_vec_to_f32(Ds + (size_t)row * hd, gd + off, u);
    }
    for (int e = threadIdx.x; e < hpc * a.topk; e += blockDim.x) {
        const int j = e % a.topk;
        const int s = a.idx[(b * a.R + r) * a.topk + j];
        const bool ok = s >= 0 && s < a.R;
        if (!ok && hg == 0 && e < a.topk) flag_error(a.err, kErrIndex);
        sreg[e] = ok ? s : -1;
    }
    __syncthreads();

    float qv[HDMAX], dov[HDMAX], dq[HDMAX];
#pragma unroll
    for (int c = 0; c < HDMAX; ++c) {
        qv[c] = (active && c < hd) ? Qs[((size_t)hl * rs + t) * hd + c] : 0.f;
        dov[c] = (active && c < hd) ? Ds[((size_t)hl * rs + t) * hd + c] : 0.f;
        dq[c] = 0.f;
    }
    // running max and sum of the softmax, and sum_i e_i (dout . v_i) relative to the same max
    float m = -INFINITY, l = 0.f, dsum = 0.f;

    // stages the key and value rows of routed slots [j0, j0 + nj) of every head of the group:
    // four 16-byte vectors of k and four of v per thread in flight before their conversion
    auto stage = [&](int j0, int nj) {
        constexpr int kBatch = 4;
        constexpr int V = Vec16<T>::N;
        const int total = hpc * nj * rs * nvh;
        for (int e0 = threadIdx.x; e0 < total; e0 += kBatch * blockDim.x) {
            uint4 kv[kBatch], vv[kBatch];
            int dsto[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                const int e = e0 + i * blockDim.x;
                dsto[i] = -1;
                if (e >= total) continue;
                const int row = e / nvh, u = e - row * nvh;
                const int eh = row / (nj * rs), key = row - eh * (nj * rs);
                const int jj = key / rs, tk = key - jj * rs;
                const int s = sreg[eh * a.topk + j0 + jj];
                if (s < 0) continue;
                const int sy = s / a.n_win, sx = s - sy * a.n_win;
                const int y = sy * a.hr + tk / a.wr, x = sx * a.wr + tk % a.wr;
                const int64_t off = ((b * a.H + y) * a.W + x) * a.C + (int64_t)(hg * hpc + eh) * hd + u * V;
                kv[i] = Vec16<T>::load_raw(gk + off);
                vv[i] = Vec16<T>::load_raw(gv + off);
                dsto[i] = (int)(eh * hstride + (size_t)key * hd + u * V);
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                if (dsto[i] >= 0) {
                    float fk[V], fv[V];
                    Vec16<T>::unpack(kv[i], fk);
                    Vec16<T>::unpack(vv[i], fv);
                    float4 *dk4 = reinterpret_cast<float4 *>(Ks + dsto[i]);
                    float4 *dv4 = reinterpret_cast<float4 *>(Vs + dsto[i]);
#pragma unroll
                    for (int j = 0; j < V / 4; ++j) {
                        dk4[j] = make_float4(fk[4 * j], fk[4 * j + 1], fk[4 * j + 2], fk[4 * j + 3]);
                        dv4[j] = make_float4(fv[4 * j], fv[4 * j + 1], fv[4 * j + 2], fv[4 * j + 3]);
                    }
                }
        }
    };

    // pass 1: the forward softmax statistics and D = dout . out = sum_i p_i (dout . v_i)
    for (int j0 = 0; j0 < a.topk; j0 += a.kcr) {
        const int nj = min(a.kcr, a.topk - j0);
        __syncthreads();
        stage(j0, nj);
        __syncthreads();
        if (!active) continue;
        for (int jj = 0; jj < nj; ++jj) {
            if (sreg[hl * a.topk + j0 + jj] < 0) continue;  // a skipped region adds no key
            for (int key = jj * rs; key < (jj + 1) * rs; ++key) {
            const float *kr = Ks + hl * hstride + (size_t)key * hd;
            const float *vr = Vs + hl * hstride + (size_t)key * hd;
            float dot = 0.f, dp = 0.f;
#pragma unroll
            for (int c = 0; c < HDMAX; ++c)
                if (c < hd) {
                    dot = fmaf(qv[c], kr[c], dot);
                    dp = fmaf(dov[c], vr[c], dp);
                }
            const float sl = dot * a.scale_log2;
            if (sl > m) {
                const float corr = fast_exp2(m - sl);
                l *= corr;
                dsum *= corr;
                m = sl;
            }
            const float p = fast_exp2(sl - m);
            l += p;
            dsum = fmaf(p, dp, dsum);
            }
        }
    }
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const float D = dsum * inv_l;

    // pass 2: p and ds per key, dq in registers; dk and dv per chunk through shared memory
    for (int j0 = 0; j0 < a.topk; j0 += a.kcr) {
        const int nj = min(a.kcr, a.topk - j0);
        __syncthreads();
        stage(j0, nj);
        __syncthreads();
        if (active) {
            for (int jj = 0; jj < nj; ++jj) {
            const bool region_ok = sreg[hl * a.topk + j0 + jj] >= 0;
            for (int key = jj * rs; key < (jj + 1) * rs; ++key) {
                float p = 0.f, ds = 0.f;
                if (region_ok) {
                    const float *kr = Ks + hl * hstride + (size_t)key * hd;
                    const float *vr = Vs + hl * hstride + (size_t)key * hd;
                    float dot = 0.f, dp = 0.f;
#pragma unroll
                    for (int c = 0; c < HDMAX; ++c)
                        if (c < hd) {
                            dot = fmaf(qv[c], kr[c], dot);
                            dp = fmaf(dov[c], vr[c], dp);
                        }
                    p = fast_exp2(dot * a.scale_log2 - m) * inv_l;
                    ds = p * (dp - D);
#pragma unroll
                    for (int c = 0; c < HDMAX; ++c)
                        if (c < hd) dq[c] = fmaf(ds, kr[c], dq[c]);
                }
                Ps[((size_t)hl * kc + key) * rs + t] = p;
                Ss[((size_t)hl * kc + key) * rs + t] = ds;
            }
            }
        }
        __syncthreads();
        // dk and dv of the chunk's keys: one thread per (head, key, 4 channels), summed over the
        // region's queries
        const int c4n = hd / 4;
        for (int e = threadIdx.x; e < hpc * nj * rs * c4n; e += blockDim.x) {
            const int eh = e / (nj * rs * c4n), rem = e - eh * (nj * rs * c4n);
            const int key = rem / c4n, c = 4 * (rem - key * c4n);
            const int jj = key / rs, tk = key - jj * rs;
            const int s = sreg[eh * a.topk + j0 + jj];
            if (s < 0) continue;
            const float *pk = Ps + ((size_t)eh * kc + key) * rs, *sk = Ss + ((size_t)eh * kc + key) * rs;
            float4 gk4 = make_float4(0.f, 0.f, 0.f, 0.f), gv4 = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int tq = 0; tq < rs; ++tq) {
                const float ds = sk[tq], p = pk[tq];
                const float4 qq = *reinterpret_cast<const float4 *>(Qs + ((size_t)eh * rs + tq) * hd + c);
                const float4 dd = *reinterpret_cast<const float4 *>(Ds + ((size_t)eh * rs + tq) * hd + c);
                gk4.x = fmaf(ds, qq.x, gk4.x);
                gk4.y = fmaf(ds, qq.y, gk4.y);
                gk4.z = fmaf(ds, qq.z, gk4.z);
                gk4.w = fmaf(ds, qq.w, gk4.w);
                gv4.x = fmaf(p, dd.x, gv4.x);
                gv4.y = fmaf(p, dd.y, gv4.y);
                gv4.z = fmaf(p, dd.z, gv4.z);
                gv4.w = fmaf(p, dd.w, gv4.w);
            }
            gk4.x *= a.scale;
            gk4.y *= a.scale;
            gk4.z *= a.scale;
            gk4.w *= a.scale;
            const int sy = s / a.n_win, sx = s - sy * a.n_win;
            const int y = sy * a.hr + tk / a.wr, x = sx * a.wr + tk % a.wr;
            const int64_t off = ((b * a.H + y) * a.W + x) * a.C + (int64_t)(hg * hpc + eh) * hd + c;
            atomicAdd(reinterpret_cast<float4 *>(a.dk + off), gk4);
            atomicAdd(reinterpret_cast<float4 *>(a.dv + off), gv4);
        }
    }
    if (active) {
        const int y = ry * a.hr + t / a.wr, x = rx * a.wr + t % a.wr;
        float *dst = a.dq + ((b * a.H + y) * a.W + x) * a.C + (int64_t)h * hd;
#pragma unroll
        for (int c = 0; c < HDMAX; ++c)
            if (c < hd) dst[c] = dq[c] * a.scale;
    }
}

// ------------------------------------------------------------------ 64-token regions, hd = 32
//
// A register-tiled variant for regions of 64 tokens and heads of 32 channels (the shape of the
// stage-1 and high-resolution workloads): one CTA of 256 threads per (image, query region,
// head); the keys arrive one routed region (64 keys) at a time. The same sums as above, as five
// 64 x 64 x 32 products on CUDA cores in fp32, each with a thread mapping whose shared-memory
// reads are broadcasts or conflict-free:
//   S, dP  : warp w owns query rows 8w .. 8w+7, lane l keys l and l + 32; q and dout are read
//            transposed (one 16-byte broadcast per 4 rows), k and v transposed (consecutive
//            keys across the lanes). A row's 64 keys sit in one warp, so its max and sums are
//            warp reductions.
//   dQ     : lane l owns rows l and l + 32, warp w channels 4w .. 4w+3: ds transposed (padded
//            rows) and k by rows (a 16-byte broadcast); dq accumulates in registers over all the
//            routed regions and is stored once.
//   dK, dV : warps 0-3 form dk, warps 4-7 dv; thread t of a half owns channels 4 (t % 8) .. + 3
//            of keys 4 (t / 8) .. + 3: ds (or p) and q (or dout) by rows, 16-byte loads; the sums
//            over the region's queries go to dk and dv with one 16-byte atomic per key.
// Rows of the tiles read by rows are padded to 36 floats, so that the staging stores of
// consecutive rows fall in different banks.
// With one routed region the scores stay in registers between the statistics and the
// gradients; with more, pass 1 gathers the statistics and pass 2 recomputes them per region.
namespace {

constexpr int kTiledThreads = 256;

// floats of each shared-memory array of the tiled kernel
constexpr int kT64 = 64 * 32;        // a 64 x 32 tile, transposed ([32][64])
constexpr int kRow = 36;             // row stride of a 64 x 32 tile kept by rows
constexpr int kTN = 64 * kRow;       // a 64 x 32 tile by rows, padded
constexpr int kTPS = 64 * 64;        // a 64 x 64 tile
constexpr int kTdSt = 64 * 65;       // transposed ds, rows padded to 65
constexpr size_t kTiledSmem = sizeof(float) * (4 * kT64 + 3 * kTN + 2 * kTPS + kTdSt) + 16 * sizeof(int);

// Loads one 64-token x 32-channel head tile (rows of the region at (y0, x0), channel offset
// c0) as fp32: into `tr` transposed ([32][64]) and, when `nat` is set, by rows ([64][kRow]).
template <typename T>
__device__ __forceinline__ void stage_head_tile(const T *g, const BackArgs &a, int64_t b, int y0, int x0, int c0,
                                                float *tr, float *nat)
{
    constexpr int V = Vec16<T>::N;  // channels per 16-byte vector
    constexpr int NV = 32 / V;      // vectors per row
    for (int e = threadIdx.x; e < 64 * NV; e += kTiledThreads) {
        const int row = e & 63, u = e >> 6;  // consecutive lanes: consecutive rows
        const int y = y0 + row / a.wr, x = x0 + row % a.wr;
        float f[V];
        Vec16<T>::load(g + ((b * a.H + y) * a.W + x) * a.C + c0 + u * V, f);
#pragma unroll
        for (int i = 0; i < V; ++i) tr[(u * V + i) * 64 + row] = f[i];
        if (nat) {
            float4 *d = reinterpret_cast<float4 *>(nat + row * kRow + u * V);
#pragma unroll
            for (int i = 0; i < V / 4; ++i) d[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        }
    }
}

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kTiledThreads, 2) attend_backward_tiled_kernel(const BackArgs a)
{
    extern __shared__ float4 smem4[];
    float *Qt = reinterpret_cast<float *>(smem4);  // [32][64] q transposed
    float *Qn = Qt + kT64;                         // [64][kRow] q
    float *Dt = Qn + kTN;                          // [32][64] dout transposed
    float *Dn = Dt + kT64;                         // [64][kRow] dout
    float *Kt = Dn + kTN;                          // [32][64] k of the routed region, transposed
    float *Kn = Kt + kT64;                         // [64][kRow] k
    float *Vt = Kn + kTN;                          // [32][64] v transposed
    float *Ps = Vt + kT64;                         // [64 queries][64 keys] p
    float *Ss = Ps + kTPS;                         // [64 queries][64 keys] ds
    float *St = Ss + kTPS;                         // [64 keys][65] ds transposed
    int *sreg = reinterpret_cast<int *>(St + kTdSt);  // routed regions (topk <= 16 staged here)

    int64_t blk = blockIdx.x;
    const int h = (int)(blk % a.heads);
    blk /= a.heads;
    const int r = (int)(blk % a.R);
    const int64_t b = blk / a.R;
    const int ry = r / a.n_win, rx = r - ry * a.n_win;
    const int c0 = h * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T *gq = static_cast<const T *>(a.q), *gk = static_cast<const T *>(a.k);
    const T *gv = static_cast<const T *>(a.v), *gd = static_cast<const T *>(a.dout);
    grid_dependency_wait();

    stage_head_tile(gq, a, b, ry * a.hr, rx * a.wr, c0, Qt, Qn);
    stage_head_tile(gd, a, b, ry * a.hr, rx * a.wr, c0, Dt, Dn);
    auto region = [&](int j) -> int {
        const int s = j < 16 ? sreg[j] : a.idx[(b * a.R + r) * a.topk + j];
        return (s >= 0 && s < a.R) ? s : -1;
    };
    if (threadIdx.x < 16 && threadIdx.x < a.topk) {
        const int s = a.idx[(b * a.R + r) * a.topk + threadIdx.x];
        sreg[threadIdx.x] = s;
    }
    if (h == 0 && threadIdx.x == 0)
        for (int j = 0; j < a.topk; ++j) {
            const int s = a.idx[(b * a.R + r) * a.topk + j];
            if (s < 0 || s >= a.R) flag_error(a.err, kErrIndex);
        }
    __syncthreads();

    // S and dP of this thread's 8 rows x 2 keys against the staged region
    float sc[8][2], dp[8][2];
    auto scores = [&]() {
#pragma unroll
        for (int i = 0; i < 8; ++i) sc[i][0] = sc[i][1] = dp[i][0] = dp[i][1] = 0.f;
#pragma unroll 4
        for (int c = 0; c < 32; ++c) {
            const float4 qa = *reinterpret_cast<const float4 *>(Qt + c * 64 + 8 * warp);
            const float4 qb = *reinterpret_cast<const float4 *>(Qt + c * 64 + 8 * warp + 4);
            const float4 da = *reinterpret_cast<const float4 *>(Dt + c * 64 + 8 * warp);
            const float4 db = *reinterpret_cast<const float4 *>(Dt + c * 64 + 8 * warp + 4);
            const float k0 = Kt[c * 64 + lane], k1 = Kt[c * 64 + lane + 32];
            const float v0 = Vt[c * 64 + lane], v1 = Vt[c * 64 + lane + 32];
            const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
            const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                sc[i][0] = fmaf(qv[i], k0, sc[i][0]);
                sc[i][1] = fmaf(qv[i], k1, sc[i][1]);
                dp[i][0] = fmaf(dv[i], v0, dp[i][0]);
                dp[i][1] = fmaf(dv[i], v1, dp[i][1]);
            }
        }
    };
    auto stage_kv = [&](int s) {
        const int sy = (s / a.n_win) * a.hr, sx = (s % a.n_win) * a.wr;
        stage_head_tile(gk, a, b, sy, sx, c0, Kt, Kn);
        stage_head_tile(gv, a, b, sy, sx, c0, Vt, static_cast<float *>(nullptr));
    };

    // pass 1: running max, sum and sum_i e_i (dout . v_i) of each of the warp's rows
    float m[8], l[8], dsum[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
        dsum[i] = 0.f;
    }
    int staged = -1;  // routed slot whose k and v are in shared memory
    for (int j = 0; j < a.topk; ++j) {
        const int s = region(j);
        if (s < 0) continue;
        __syncthreads();
        stage_kv(s);
        staged = j;
        __syncthreads();
        scores();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float s0 = sc[i][0] * a.scale_log2, s1 = sc[i][1] * a.scale_log2;
            const float mn = fmaxf(m[i], warp_max(fmaxf(s0, s1)));
            const float corr = fast_exp2(m[i] - mn);
            const float e0 = fast_exp2(s0 - mn), e1 = fast_exp2(s1 - mn);
            l[i] = l[i] * corr + warp_sum(e0 + e1);
            dsum[i] = dsum[i] * corr + warp_sum(fmaf(e0, dp[i][0], e1 * dp[i][1]));
            m[i] = mn;
        }
    }
    float inv_l[8], D[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        inv_l[i] = l[i] > 0.f ? 1.f / l[i] : 0.f;
        D[i] = dsum[i] * inv_l[i];
    }

    // pass 2: p and ds per routed region; dq in registers, dk and dv added per region
    float dq[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
    // dK (warps 0-3) or dV (warps 4-7): keys 4 kg .. + 3, channels 4 c4 .. + 3
    const int half = warp >> 2, ht = threadIdx.x & 127;
    const int c4 = ht & 7, kg = ht >> 3;
    for (int j = 0; j < a.topk; ++j) {
        const int s = region(j);
        if (s < 0) continue;
        if (staged != j) {  // the last region of pass 1 is still staged, its scores in registers
            __syncthreads();
            stage_kv(s);
            __syncthreads();
            scores();
        }
        staged = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int row = 8 * warp + i;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int key = lane + 32 * t;
                const float p = fast_exp2(fmaf(sc[i][t], a.scale_log2, -m[i])) * inv_l[i];
                const float ds = p * (dp[i][t] - D[i]);
                Ps[row * 64 + key] = p;
                Ss[row * 64 + key] = ds;
                St[key * 65 + row] = ds;
            }
        }
        __syncthreads();
        // dq rows lane, lane + 32, channels 4 warp ..: sum over the region's 64 keys
#pragma unroll 4
        for (int key = 0; key < 64; ++key) {
            const float4 kr = *reinterpret_cast<const float4 *>(Kn + key * kRow + 4 * warp);
            const float d0 = St[key * 65 + lane], d1 = St[key * 65 + lane + 32];
            dq[0][0] = fmaf(d0, kr.x, dq[0][0]);
            dq[0][1] = fmaf(d0, kr.y, dq[0][1]);
            dq[0][2] = fmaf(d0, kr.z, dq[0][2]);
            dq[0][3] = fmaf(d0, kr.w, dq[0][3]);
            dq[1][0] = fmaf(d1, kr.x, dq[1][0]);
            dq[1][1] = fmaf(d1, kr.y, dq[1][1]);
            dq[1][2] = fmaf(d1, kr.z, dq[1][2]);
            dq[1][3] = fmaf(d1, kr.w, dq[1][3]);
        }
        // dk (or dv) of keys 4 kg .. + 3, channels 4 c4 ..: sums over the region's 64 queries of
        // ds q (or p dout)
        {
            const float *coef = half ? Ps : Ss;
            const float *rows = half ? Dn : Qn;
            float4 g4[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) g4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int row = 0; row < 64; ++row) {
                const float4 x = *reinterpret_cast<const float4 *>(rows + row * kRow + 4 * c4);
                const float4 w4 = *reinterpret_cast<const float4 *>(coef + row * 64 + 4 * kg);
                const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    g4[t].x = fmaf(wv[t], x.x, g4[t].x);
                    g4[t].y = fmaf(wv[t], x.y, g4[t].y);
                    g4[t].z = fmaf(wv[t], x.z, g4[t].z);
                    g4[t].w = fmaf(wv[t], x.w, g4[t].w);
                }
            }
            const int sy = (s / a.n_win) * a.hr, sx = (s % a.n_win) * a.wr;
            const float sc4 = half ? 1.f : a.scale;
            float *dst = half ? a.dv : a.dk;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int key = 4 * kg + t;
                const int y = sy + key / a.wr, x = sx + key % a.wr;
                const int64_t off = ((b * a.H + y) * a.W + x) * a.C + c0 + 4 * c4;
                atomicAdd(reinterpret_cast<float4 *>(dst + off),
                          make_float4(g4[t].x * sc4, g4[t].y * sc4, g4[t].z * sc4, g4[t].w * sc4));
            }
        }
        __syncthreads();  // p and ds are rewritten by the next region
    }
    const int y0 = ry * a.hr, x0 = rx * a.wr;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int row = lane + 32 * i;
        const int y = y0 + row / a.wr, x = x0 + row % a.wr;
        float *dst = a.dq + ((b * a.H + y) * a.W + x) * a.C + c0 + 4 * warp;
        *reinterpret_cast<float4 *>(dst) =
            make_float4(dq[i][0] * a.scale, dq[i][1] * a.scale, dq[i][2] * a.scale, dq[i][3] * a.scale);
    }
}

// ------------------------------------------------------------------ tensor cores, bf16
//
// The same gradients for bf16 inputs of 64-token regions and 32-channel heads on mma.sync
// (m16n8k16, fp32 accumulation), a persistent grid of CTAs of 4 warps, each taking (image, query
// region, head) items in turn:
//   S = Q K^T and dP = dout V^T take the bf16 inputs as they are (their products are exact in
//   fp32); P and dS are fp32 and enter the three products that use them as two bf16 terms,
//   x = hi + lo with hi = x with its low 16 bits cleared (exact) and lo = x - hi rounded to bf16,
//   so that each such operand carries about 16 significant bits (relative error <= 2^-16)
//   and every product is again exact in fp32:
//   dQ = dS K          (A = the warp's 16 query rows of dS, B = K),
//   dK = dS^T Q, dV = P^T dout (A = dS^T, P^T read transposed from shared memory, B = Q, dout).
// ds and then p pass through one pair of shared arrays (high and low part) and dq accumulates
// in shared memory. The next item's q and dout tiles, and k and v of its first routed region,
// arrive by cp.async in a second set of tiles while the CTA works on the current item, so that
// the loads' latency is hidden; with the two sets a CTA needs 68 KB, and three share an SM.
// Warp w owns query rows 16w .. 16w+15 for S, dP and dQ, and key rows 16w .. 16w+15 of each
// routed region for dK and dV. Row statistics (running max, sum, D = sum p dp) are quad
// reductions; with one routed region the scores stay in registers between the passes.
namespace {

constexpr int kMmaBackWarps = 4;
constexpr int kTileRow = 40;   // bf16 per row of a 64 x 32 tile (32 + 8: rows 80 bytes apart)
constexpr int kPRow = 72;      // bf16 per row of a 64 x 64 tile of p or ds (64 + 8)
constexpr int kDqRow = 40;     // fp32 per row of the 64 x 32 dq accumulator (32 + 8)
constexpr int kMmaBackCtasPerSm = 3;
constexpr size_t kMmaBackSmem = sizeof(__nv_bfloat16) * (2 * 4 * 64 * kTileRow + 2 * 64 * kPRow) +
                                sizeof(float) * 64 * kDqRow + 2 * 16 * sizeof(int);

__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const float h0 = bf16_trunc(x0), h1 = bf16_trunc(x1);
    hi = pack_bf16x2_trunc(h0, h1);
    lo = pack_bf16x2(x0 - h0, x1 - h1);
}

__device__ __forceinline__ float quad_max_b(float x)
{
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ float quad_sum_b(float x)
{
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// One 64-token x 32-channel bf16 head tile of the region at (y0, x0), channel offset c0, into
// shared memory rows of kTileRow bf16 (16-byte vectors, all threads).
__device__ __forceinline__ void stage_bf16_tile(const __nv_bfloat16 *g, const BackArgs &a, int64_t b, int y0, int x0,
                                                int c0, __nv_bfloat16 *dst)
{
    for (int e = threadIdx.x; e < 64 * 4; e += 32 * kMmaBackWarps) {
        const int row = e >> 2, u = e & 3;
        const int y = y0 + row / a.wr, x = x0 + row % a.wr;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(g + ((b * a.H + y) * a.W + x) * a.C + c0 + 8 * u));
        *reinterpret_cast<uint4 *>(dst + row * kTileRow + 8 * u) = v;
    }
}

// The same tile as stage_bf16_tile, by asynchronous copies that land while the CTA computes
__device__ __forceinline__ void fetch_bf16_tile(const __nv_bfloat16 *g, const BackArgs &a, int64_t b, int y0, int x0,
                                                int c0, __nv_bfloat16 *dst)
{
    for (int e = threadIdx.x; e < 64 * 4; e += 32 * kMmaBackWarps) {
        const int row = e >> 2, u = e & 3;
        const int y = y0 + row / a.wr, x = x0 + row % a.wr;
        cp_async16(smem_u32(dst + row * kTileRow + 8 * u), g + ((b * a.H + y) * a.W + x) * a.C + c0 + 8 * u);
    }
}

}  // namespace

__global__ void __launch_bounds__(32 * kMmaBackWarps, kMmaBackCtasPerSm) attend_backward_mma_kernel(const BackArgs a)
{
    extern __shared__ float4 smem4[];
    // two sets of [q, dout, k, v] tiles of [64][kTileRow]: the CTA works on one item while the
    // next item's tiles land in the other
    __nv_bfloat16 *tiles = reinterpret_cast<__nv_bfloat16 *>(smem4);
    __nv_bfloat16 *sPh = tiles + 8 * 64 * kTileRow;                 // [64 queries][kPRow] ds, then p: high part
    __nv_bfloat16 *sPl = sPh + 64 * kPRow;                          // low part
    float *sDq = reinterpret_cast<float *>(sPl + 64 * kPRow);       // [64 queries][kDqRow] dq accumulator
    int *sregs = reinterpret_cast<int *>(sDq + 64 * kDqRow);        // [2][16] routed regions of each set's item

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    float *const dq_own = sDq + (16 * warp + g) * kDqRow + 2 * t;  // this thread's dq: rows g, g + 8
    const __nv_bfloat16 *gq = static_cast<const __nv_bfloat16 *>(a.q), *gk = static_cast<const __nv_bfloat16 *>(a.k);
    const __nv_bfloat16 *gv = static_cast<const __nv_bfloat16 *>(a.v), *gd = static_cast<const __nv_bfloat16 *>(a.dout);
    // item = (image b, query region r, head h), heads fastest; its index row is item / heads
    auto fetch_qd = [&](int item, int set) {
        const int h = item % a.heads, r = (item / a.heads) % a.R;
        const int64_t b = (item / a.heads) / a.R;
        const int ry = r / a.n_win, rx = r - ry * a.n_win;
        __nv_bfloat16 *base = tiles + set * 4 * 64 * kTileRow;
        fetch_bf16_tile(gq, a, b, ry * a.hr, rx * a.wr, h * 32, base);
        fetch_bf16_tile(gd, a, b, ry * a.hr, rx * a.wr, h * 32, base + 64 * kTileRow);
    };
    auto fetch_kv = [&](int item, int s, int set) {
        const int h = item % a.heads;
        const int64_t b = (item / a.heads) / a.R;
        __nv_bfloat16 *base = tiles + set * 4 * 64 * kTileRow + 2 * 64 * kTileRow;
        fetch_bf16_tile(gk, a, b, (s / a.n_win) * a.hr, (s % a.n_win) * a.wr, h * 32, base);
        fetch_bf16_tile(gv, a, b, (s / a.n_win) * a.hr, (s % a.n_win) * a.wr, h * 32, base + 64 * kTileRow);
    };
    auto idx_at = [&](int item, int j) -> int { return __ldg(a.idx + (int64_t)(item / a.heads) * a.topk + j); };
    grid_dependency_wait();

    int item = blockIdx.x;
    if (item >= a.nitems) return;
    {  // the first item: its tiles into set 0 (k and v of its first routed region, when valid)
        const int s0 = idx_at(item, 0);
        if (threadIdx.x < 16 && threadIdx.x < a.topk) sregs[threadIdx.x] = idx_at(item, threadIdx.x);
        fetch_qd(item, 0);
        if (s0 >= 0 && s0 < a.R) fetch_kv(item, s0, 0);
        cp_async_commit();
    }
    for (int cur = 0;; cur ^= 1) {
        const int64_t next64 = (int64_t)item + gridDim.x;
        const bool has_next = next64 < a.nitems;
        const int next = has_next ? (int)next64 : 0;
        // the next item's index entries: loaded now, used once pass 1 is done
        int s_next = -1, reg_next = 0;
        if (has_next) {
            s_next = idx_at(next, 0);
            if (threadIdx.x < 16 && threadIdx.x < a.topk) reg_next = idx_at(next, threadIdx.x);
        }
        cp_async_wait_all();
        __syncthreads();  // this item's tiles are in place; the other set is free
        if (has_next) fetch_qd(next, cur ^ 1);
        cp_async_commit();

        const int h = item % a.heads;
        const int r = (item / a.heads) % a.R;
        const int64_t b = (item / a.heads) / a.R;
        const int ry = r / a.n_win, rx = r - ry * a.n_win;
        const int c0 = h * 32;
        const int *sreg = sregs + 16 * cur;
        __nv_bfloat16 *sQ = tiles + cur * 4 * 64 * kTileRow;
        __nv_bfloat16 *sD = sQ + 64 * kTileRow, *sK = sD + 64 * kTileRow, *sV = sK + 64 * kTileRow;
        if (h == 0 && threadIdx.x == 0)
            for (int j = 0; j < a.topk; ++j) {
                const int s = j < 16 ? sreg[j] : a.idx[(b * a.R + r) * a.topk + j];
                if (s < 0 || s >= a.R) flag_error(a.err, kErrIndex);
            }
        auto region = [&](int j) -> int {
            const int s = j < 16 ? sreg[j] : a.idx[(b * a.R + r) * a.topk + j];
            return (s >= 0 && s < a.R) ? s : -1;
        };

        // shared-memory addresses of the tiles; the A fragments of q and dout are read per score pass
        const uint32_t q0 = smem_u32(sQ), d0 = smem_u32(sD), k0 = smem_u32(sK), v0 = smem_u32(sV);

        // S and dP of the warp's rows against the staged region: 8 key tiles of 8
        float sc[8][4], dp[8][4];
        auto scores = [&]() {
            uint32_t qf[2][4], df[2][4];
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const uint32_t off = (uint32_t)((16 * warp + (lane & 15)) * kTileRow + 16 * ks + 8 * (lane >> 4)) * 2u;
                ldmatrix_x4(q0 + off, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
                ldmatrix_x4(d0 + off, df[ks][0], df[ks][1], df[ks][2], df[ks][3]);
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                dp[nt][0] = dp[nt][1] = dp[nt][2] = dp[nt][3] = 0.f;
                const uint32_t off = (uint32_t)((8 * nt + (lane & 7)) * kTileRow + 8 * (lane >> 3)) * 2u;
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(k0 + off, b0, b1, b2, b3);
                mma_bf16_16816(sc[nt], qf[0], b0, b1);
                mma_bf16_16816(sc[nt], qf[1], b2, b3);
                ldmatrix_x4(v0 + off, b0, b1, b2, b3);
                mma_bf16_16816(dp[nt], df[0], b0, b1);
                mma_bf16_16816(dp[nt], df[1], b2, b3);
            }
        };
        auto stage_kv = [&](int s) {
            const int sy = (s / a.n_win) * a.hr, sx = (s % a.n_win) * a.wr;
            stage_bf16_tile(gk, a, b, sy, sx, c0, sK);
            stage_bf16_tile(gv, a, b, sy, sx, c0, sV);
        };

        // pass 1: running max, sum and sum e (dout . v) of rows g and g + 8
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, dsum[2] = {0.f, 0.f};
        int staged = -1;
        for (int j = 0; j < a.topk; ++j) {
            const int s = region(j);
            if (s < 0) continue;
            if (j != 0) {  // the first routed region came with the item's tiles
                __syncthreads();
                stage_kv(s);
                __syncthreads();
            }
            staged = j;
            scores();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float mx = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(sc[nt][2 * hh], sc[nt][2 * hh + 1]));
                const float mn = fmaxf(m[hh], quad_max_b(mx) * a.scale_log2);
                const float corr = fast_exp2(m[hh] - mn);
                float es = 0.f, eds = 0.f;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float e = fast_exp2(fmaf(sc[nt][2 * hh + i], a.scale_log2, -mn));
                        es += e;
                        eds = fmaf(e, dp[nt][2 * hh + i], eds);
                    }
                l[hh] = l[hh] * corr + quad_sum_b(es);
                dsum[hh] = dsum[hh] * corr + quad_sum_b(eds);
                m[hh] = mn;
            }
        }
        // the next item's first routed region into the other set, and its index entries
        if (has_next && s_next >= 0 && s_next < a.R) fetch_kv(next, s_next, cur ^ 1);
        cp_async_commit();
        if (has_next && threadIdx.x < 16 && threadIdx.x < a.topk) sregs[16 * (cur ^ 1) + threadIdx.x] = reg_next;
        float inv_l[2], D[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            inv_l[hh] = l[hh] > 0.f ? 1.f / l[hh] : 0.f;
            D[hh] = dsum[hh] * inv_l[hh];
        }

        // pass 2: p and ds per routed region; dq in shared memory (each warp its own rows), dk and dv
        // added per region
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
                *reinterpret_cast<float2 *>(dq_own + 8 * hh * kDqRow + 8 * nt) = make_float2(0.f, 0.f);
        for (int j = 0; j < a.topk; ++j) {
            const int s = region(j);
            if (s < 0) continue;
            if (staged != j) {
                __syncthreads();
                stage_kv(s);
                __syncthreads();
                scores();
            }
            staged = -1;
            // p and ds in place of the scores; their bf16 high and low parts to shared memory
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int hh = i >> 1;
                    const float p = fast_exp2(fmaf(sc[nt][i], a.scale_log2, -m[hh])) * inv_l[hh];
                    sc[nt][i] = p;
                    dp[nt][i] = p * (dp[nt][i] - D[hh]);
                }
            const int sy = (s / a.n_win) * a.hr, sx = (s % a.n_win) * a.wr;
            const int mrow = (lane >> 4) & 1, mcol = (lane >> 3) & 1;  // which 8 x 8 of the 16 x 16 A tile
            // ds, then p, through one pair of shared arrays (high and low part): dQ += dS K (A = the
            // warp's own rows of ds), dK = dS^T Q, then dV = P^T dout
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = 16 * warp + g + 8 * hh, col = 8 * nt + 2 * t;
                        uint32_t hi, lo;
                        if (pass == 0)
                            split_pack(dp[nt][2 * hh], dp[nt][2 * hh + 1], hi, lo);
                        else
                            split_pack(sc[nt][2 * hh], sc[nt][2 * hh + 1], hi, lo);
                        *reinterpret_cast<uint32_t *>(sPh + row * kPRow + col) = hi;
                        *reinterpret_cast<uint32_t *>(sPl + row * kPRow + col) = lo;
                    }
                __syncthreads();
                if (pass == 0) {
                    float dq[4][4];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int nt = 0; nt < 4; ++nt) {
                            const float2 v2 = *reinterpret_cast<const float2 *>(dq_own + 8 * hh * kDqRow + 8 * nt);
                            dq[nt][2 * hh] = v2.x;
                            dq[nt][2 * hh + 1] = v2.y;
                        }
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t aoff =
                            (uint32_t)((16 * warp + (lane & 15)) * kPRow + 16 * kk + 8 * (lane >> 4)) * 2u;
                        uint32_t ah[4], al[4];
                        ldmatrix_x4(smem_u32(sPh) + aoff, ah[0], ah[1], ah[2], ah[3]);
                        ldmatrix_x4(smem_u32(sPl) + aoff, al[0], al[1], al[2], al[3]);
#pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            const int row = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4_trans(k0 + (uint32_t)(row * kTileRow + 16 * np + 8 * (lane >> 4)) * 2u,
                                              b0, b1, b2, b3);
                            mma_bf16_16816(dq[2 * np], al, b0, b1);
                            mma_bf16_16816(dq[2 * np + 1], al, b2, b3);
                            mma_bf16_16816(dq[2 * np], ah, b0, b1);
                            mma_bf16_16816(dq[2 * np + 1], ah, b2, b3);
                        }
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int nt = 0; nt < 4; ++nt)
                            *reinterpret_cast<float2 *>(dq_own + 8 * hh * kDqRow + 8 * nt) =
                                make_float2(dq[nt][2 * hh], dq[nt][2 * hh + 1]);
                }
                float g4[4][4];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) g4[nt][0] = g4[nt][1] = g4[nt][2] = g4[nt][3] = 0.f;
                const uint32_t bbase = pass == 0 ? q0 : d0;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {  // 16 queries per step
                    const uint32_t aoff =
                        (uint32_t)((16 * kk + (lane & 7) + 8 * mrow) * kPRow + 16 * warp + 8 * mcol) * 2u;
                    uint32_t ah[4], al[4];
                    ldmatrix_x4_trans(smem_u32(sPh) + aoff, ah[0], ah[1], ah[2], ah[3]);
                    ldmatrix_x4_trans(smem_u32(sPl) + aoff, al[0], al[1], al[2], al[3]);
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        const int row = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4_trans(bbase + (uint32_t)(row * kTileRow + 16 * np + 8 * (lane >> 4)) * 2u,
                                          b0, b1, b2, b3);
                        mma_bf16_16816(g4[2 * np], al, b0, b1);
                        mma_bf16_16816(g4[2 * np + 1], al, b2, b3);
                        mma_bf16_16816(g4[2 * np], ah, b0, b1);
                        mma_bf16_16816(g4[2 * np + 1], ah, b2, b3);
                    }
                }
                const float sc4 = pass == 0 ? a.scale : 1.f;
                float *dst = pass == 0 ? a.dk : a.dv;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int key = 16 * warp + g + 8 * hh;
                    const int y = sy + key / a.wr, x = sx + key % a.wr;
                    const int64_t off = ((b * a.H + y) * a.W + x) * a.C + c0 + 2 * t;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
                        atomicAdd(reinterpret_cast<float2 *>(dst + off + 8 * nt),
                                  make_float2(g4[nt][2 * hh] * sc4, g4[nt][2 * hh + 1] * sc4));
                }
                __syncthreads();  // the arrays are rewritten next
            }
        }
        const int y0 = ry * a.hr, x0 = rx * a.wr;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = 16 * warp + g + 8 * hh;
            const int y = y0 + row / a.wr, x = x0 + row % a.wr;
            float *dst = a.dq + ((b * a.H + y) * a.W + x) * a.C + c0 + 2 * t;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float2 v2 = *reinterpret_cast<const float2 *>(dq_own + 8 * hh * kDqRow + 8 * nt);
                *reinterpret_cast<float2 *>(dst + 8 * nt) = make_float2(v2.x * a.scale, v2.y * a.scale);
            }
        }
        if (!has_next) break;
        item = next;
    }
}

namespace {

constexpr size_t kBackMaxSmem = 100 * 1024;

size_t back_smem(int hpc, int rs, int hd, int kcr, int topk)
{
    const size_t kc = (size_t)kcr * rs;
    return sizeof(float) * ((size_t)2 * hpc * rs * hd + (size_t)2 * hpc * (kc * hd + 4) + (size_t)2 * hpc * rs * kc) +
           4 * (size_t)hpc * topk + 16;
}

}  // namespace

bool attend_backward_supports(const Geometry &g)
{
    // a head row is a whole number of 16-byte vectors of bf16 (hd % 8) and of fp32 (hd % 4)
    return g.rs <= 256 && g.hd % 8 == 0 && g.hd <= kSimtMaxHeadDim && back_smem(1, g.rs, g.hd, 1, g.topk) <= kBackMaxSmem;
}

cudaError_t launch_attend_backward(const void *q, const void *k, const void *v, const int32_t *idx, const void *dout,
                                   float *dq, float *dk, float *dv, const Geometry &g, bool bf16, unsigned *err,
                                   cudaStream_t stream)
{
    if (!attend_backward_supports(g)) return cudaErrorInvalidConfiguration;
    BackArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.dout = dout;
    a.idx = idx;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.err = err;
    a.H = g.H;
    a.W = g.W;
    a.C = g.C;
    a.heads = g.heads;
    a.hd = g.hd;
    a.n_win = g.n_win;
    a.hr = g.hr;
    a.wr = g.wr;
    a.rs = g.rs;
    a.R = g.R;
    a.topk = g.topk;
    a.scale = (float)(1.0 / sqrt((double)g.hd));
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    if (g.rs == 64 && g.hd == 32 && bf16) {
        // 64-token regions, heads of 32 channels, bf16: the persistent tensor-core kernel
        const long long items = (long long)g.B * g.R * g.heads;
        if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        a.nitems = (int)items;
        const size_t bytes = (size_t)g.B * g.H * g.W * g.C * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dk, 0, bytes, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, stream);
        if (e != cudaSuccess) return e;
        static int granted_mma[64] = {0};
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        int sms = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        const long long blocks = std::min(items, (long long)kMmaBackCtasPerSm * std::max(sms, 1));
        if ((int)kMmaBackSmem > 48 * 1024 && (int)kMmaBackSmem > granted_mma[dev]) {
            if ((e = cudaFuncSetAttribute(attend_backward_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kMmaBackSmem)) != cudaSuccess)
                return e;
            granted_mma[dev] = (int)kMmaBackSmem;
        }
        return launch_pdl(attend_backward_mma_kernel, dim3((unsigned)blocks), dim3(32 * kMmaBackWarps), kMmaBackSmem,
                          stream, a);
    }
    if (g.rs == 64 && g.hd == 32) {
        // 64-token regions, heads of 32 channels, fp32: the register-tiled kernel
        const long long blocks = (long long)g.B * g.R * g.heads;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        const size_t bytes = (size_t)g.B * g.H * g.W * g.C * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dk, 0, bytes, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, stream);
        if (e != cudaSuccess) return e;
        void (*kernel)(const BackArgs) = attend_backward_tiled_kernel<float>;
        static int granted_tiled[64] = {0};
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if ((int)kTiledSmem > granted_tiled[dev]) {
            if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTiledSmem)) !=
                cudaSuccess)
                return e;
            granted_tiled[dev] = (int)kTiledSmem;
        }
        return launch_pdl(kernel, dim3((unsigned)blocks), dim3(kTiledThreads), kTiledSmem, stream, a);
    }
    // heads per CTA: the largest divisor of heads with hpc * rs <= 256 threads whose smem holds at
    // least one routed region per chunk; then as many regions per chunk as fit
    int hpc = 1;
    for (int d = 1; d <= g.heads; ++d)
        if (g.heads % d == 0 && (long long)d * g.rs <= 256 && back_smem(d, g.rs, g.hd, 1, g.topk) <= kBackMaxSmem)
            hpc = d;
    int kcr = 1;
    while (kcr < g.topk && back_smem(hpc, g.rs, g.hd, kcr + 1, g.topk) <= kBackMaxSmem) ++kcr;
    a.hpc = hpc;
    a.kcr = kcr;
    const size_t smem = back_smem(hpc, g.rs, g.hd, kcr, g.topk);
    const int threads = ((hpc * g.rs + 31) / 32) * 32;
    const long long blocks = (long long)g.B * g.R * (g.heads / hpc);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const size_t bytes = (size_t)g.B * g.H * g.W * g.C * sizeof(float);
    cudaError_t e = cudaMemsetAsync(dk, 0, bytes, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, stream);
    if (e != cudaSuccess) return e;
    void (*kernel)(const BackArgs) = nullptr;
    int slot = 0;
    if (g.hd <= 32) {
        kernel = bf16 ? attend_backward_kernel<__nv_bfloat16, 32> : attend_backward_kernel<float, 32>;
        slot = bf16 ? 0 : 1;
    } else if (g.hd <= 64) {
        kernel = bf16 ? attend_backward_kernel<__nv_bfloat16, 64> : attend_backward_kernel<float, 64>;
        slot = bf16 ? 2 : 3;
    } else {
        kernel = bf16 ? attend_backward_kernel<__nv_bfloat16, 128> : attend_backward_kernel<float, 128>;
        slot = bf16 ? 4 : 5;
    }
    static int granted[6][64] = {{0}};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (smem > 48 * 1024 && (int)smem > granted[slot][dev]) {
        if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        granted[slot][dev] = (int)smem;
    }
    return launch_pdl(kernel, dim3((unsigned)blocks), dim3(threads), smem, stream, a);
}

}  // namespace bra
