// bra_attend_umma.cu -- gather attention on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators) for regions of 64 tokens and heads of 32 channels (bf16).
//
// What it computes ("从零构建BiFormer", §2.2 TokenAttention; "医学图像分割模块：BiFormer /
// 双层路由注意力", §五 steps ⑤-⑦): for every query token of region r and every head, softmax
// (scale head_dim^-1/2) over the tokens of the regions idx[b, r, 0..topk-1], then the weighted
// sum of their values, accumulated in fp32, out rounded to bf16.
//
// One work item = (image, query region, 64-channel block = 2 heads). Per CTA, 6 warps:
//  * warp 0 lane 0, producer: TMA loads of the query tile (64 tokens x 64 channels) into a
//    ring of query slots and, per routed region, of its K and V tiles into a ring of KV
//    slots (128-byte swizzle, no multicast), as in the mma.sync gather kernel;
//  * warp 1: allocates 128 TMEM columns; its lane 0 issues every MMA. Per routed region:
//      S_h = Q_h K_h^T  (M = 64 query rows, N = 64 keys, K = 32 channels of head h), head 0
//                        into TMEM lanes {0-15, 32-47, 64-79, 96-111} columns 0-63, head 1 into
//                        the same columns at lane offset 16 (an M = 64 accumulator fills 16
//                        lanes of each 32-lane quadrant);
//      O_h = P_h V      (M = 64, N = 64 channels of V, K = 64 keys), P_h from shared memory;
//                        head 0 at columns 64-127, head 1 at columns 32-95 of its lanes, so
//                        that both heads' own 32 output channels land in columns 64-95.
//    tcgen05.commit signals each product on an mbarrier and frees the query / KV slots.
//  * warps 2-5, softmax: thread t of warp w owns query row 16 (w % 4) + (t % 16) of head t / 16,
//    i.e. TMEM lane 32 (w % 4) + t. Per region it loads its 64 scores, updates the running max
//    and sum (exp2 with a log2(e) pre-scale), writes its 64 probabilities (rounded down to bf16,
//    the sum taken over exactly those values) into the P tile, then adds the region's PV
//    product into 32 fp32 registers (rescaled by the max correction). After the last region
//    it normalises and stores its 32 output channels (64 contiguous bytes).
// Every wait is bounded (kErrTimeout); no thread leaves before the TMEM is released.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

constexpr int kRows = 64;                 // tokens per region = M of every MMA
constexpr int kTile = kRows * 128;        // 64 rows x 64 bf16 channels, 128-byte swizzled rows
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kIdescS = umma_idesc_bf16(64, 64, false);  // Q K^T: B = K tile, K-major
constexpr uint32_t kIdescPV = umma_idesc_bf16(64, 64, true);  // P V: B = V tile, MN-major

struct UmmaArgs {
    const int32_t *idx;
    unsigned *err;
    __nv_bfloat16 *out;
    int H, W, C, n_win, topk, R, hr, wr;
    int ncb;  // 64-channel blocks = work items per (image, region)
    int nitems, per_cta, qslots, kvslots, idx_chunk;
    float scale_log2;
};

struct UmmaItem {
    int b, qx, qy, cb;
};

}  // namespace

__global__ void __launch_bounds__(192, 1) attend_gather_umma_kernel(const __grid_constant__ CUtensorMap tq,
                                                                    const __grid_constant__ CUtensorMap tk,
                                                                    const __grid_constant__ CUtensorMap tv,
                                                                    const UmmaArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sKV = sQ + (size_t)a.qslots * kTile;
    uint8_t *sP = sKV + (size_t)a.kvslots * 2 * kTile;  // P tiles of heads 0 and 1
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sP + 2 * kTile);
    uint64_t *q_empty = q_full + a.qslots;
    uint64_t *kv_full = q_empty + a.qslots;
    uint64_t *kv_empty = kv_full + a.kvslots;
    uint64_t *s_full = kv_empty + a.kvslots;
    uint64_t *p_full = s_full + 1;
    uint64_t *o_full = p_full + 1;
    uint64_t *o_free = o_full + 1;
    uint64_t *drain = o_free + 1;
    int *kv_ok = reinterpret_cast<int *>(drain + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(kv_ok + a.kvslots);
    int *sidx = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int begin = blockIdx.x * a.per_cta;
    const int end = min(a.nitems, begin + a.per_cta);

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.qslots; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < a.kvslots; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, 4);
        mbar_init(o_full, 1);
        mbar_init(o_free, 4);
        mbar_init(drain, 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tcgen05_before_sync();
    __syncthreads();
    tcgen05_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------- producer (TMA)
        int qs = 0, kvs = 0;
        uint32_t qph = 0, kvph = 0;
        bool alive = true;
        for (int c0 = begin; c0 < end; c0 += a.idx_chunk) {
            const int n = min(a.idx_chunk, end - c0);
            __syncwarp();
            for (int e = lane; e < n * a.topk; e += 32) {
                const int it = c0 + e / a.topk, j = e % a.topk;
                sidx[e] = a.idx[(int64_t)(it / a.ncb) * a.topk + j];
            }
            __syncwarp();
            if (lane != 0 || !alive) continue;
            for (int i = 0; i < n && alive; ++i) {
                const int item = c0 + i;
                const int cb = item % a.ncb;
                const int br = item / a.ncb;
                const int r = br % a.R, b = br / a.R;
                const int qx = (r % a.n_win) * a.wr, qy = (r / a.n_win) * a.hr;
                if (!(alive = mbar_wait(&q_empty[qs], qph ^ 1, a.err))) break;
                mbar_arrive_expect_tx(&q_full[qs], (uint32_t)kTile);
                tma_load_4d(sQ + (size_t)qs * kTile, &tq, cb * 64, qx, qy, b, &q_full[qs]);
                if (++qs == a.qslots) {
                    qs = 0;
                    qph ^= 1;
                }
                for (int j = 0; j < a.topk; ++j) {
                    const int s = sidx[i * a.topk + j];
                    const bool ok = s >= 0 && s < a.R;
                    if (!(alive = mbar_wait(&kv_empty[kvs], kvph ^ 1, a.err))) break;
                    kv_ok[kvs] = ok;
                    if (ok) {
                        const int sx = (s % a.n_win) * a.wr, sy = (s / a.n_win) * a.hr;
                        uint8_t *kt = sKV + (size_t)kvs * 2 * kTile;
                        mbar_arrive_expect_tx(&kv_full[kvs], (uint32_t)(2 * kTile));
                        tma_load_4d(kt, &tk, cb * 64, sx, sy, b, &kv_full[kvs]);
                        tma_load_4d(kt + kTile, &tv, cb * 64, sx, sy, b, &kv_full[kvs]);
                    } else {
                        flag_error(a.err, kErrIndex);
                        mbar_arrive_expect_tx(&kv_full[kvs], 0);
                    }
                    if (++kvs == a.kvslots) {
                        kvs = 0;
                        kvph ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int qs = 0, kvs = 0;
            uint32_t qph = 0, kvph = 0, pph = 0, fph = 0;
            bool alive = true, first_pv = true;
            const uint32_t p_base = smem_u32(sP);
            for (int item = begin; item < end && alive; ++item) {
                if (!(alive = mbar_wait(&q_full[qs], qph, a.err))) break;
                tcgen05_after_sync();
                const uint32_t qa = smem_u32(sQ + (size_t)qs * kTile);
                for (int j = 0; j < a.topk; ++j) {
                    if (!(alive = mbar_wait(&kv_full[kvs], kvph, a.err))) break;
                    tcgen05_after_sync();
                    const bool ok = kv_ok[kvs] != 0;
                    const uint32_t ka = smem_u32(sKV + (size_t)kvs * 2 * kTile), va = ka + kTile;
                    if (ok) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int ks = 0; ks < 2; ++ks)
                                umma_bf16(tmem + ((uint32_t)(16 * h) << 16),
                                          umma_desc_sw128(qa + h * 64 + ks * 32),
                                          umma_desc_sw128(ka + h * 64 + ks * 32), kIdescS, (uint32_t)ks);
                        umma_commit(s_full);
                    } else {
                        mbar_arrive(s_full);
                    }
                    if (j == a.topk - 1) umma_commit(&q_empty[qs]);
                    if (!(alive = mbar_wait(p_full, pph, a.err))) break;
                    pph ^= 1;
                    if (!first_pv) {
                        if (!(alive = mbar_wait(o_free, fph, a.err))) break;
                        fph ^= 1;
                    }
                    first_pv = false;
                    tcgen05_after_sync();
                    if (ok) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16(tmem + ((uint32_t)(16 * h) << 16) + (h ? 32u : 64u),
                                          umma_desc_sw128(p_base + h * kTile + kk * 32),
                                          umma_desc_sw128(va + kk * 2048), kIdescPV, (uint32_t)kk);
                        umma_commit(o_full);
                    } else {
                        mbar_arrive(o_full);
                    }
                    umma_commit(&kv_empty[kvs]);
                    if (++kvs == a.kvslots) {
                        kvs = 0;
                        kvph ^= 1;
                    }
                }
                if (++qs == a.qslots) {
                    qs = 0;
                    qph ^= 1;
                }
            }
            // every commit above arrives once the MMAs before it are done; wait for the last
            // one so that no arrival lands after this CTA has left
            umma_commit(drain);
            mbar_wait(drain, 0, a.err);
        }
    } else {
        // ------------------------------------------------------------- softmax warpgroup
        const int q = warp & 3;  // the TMEM lane quadrant this warp may access
        const int h = lane >> 4;
        const int row = 16 * q + (lane & 15);
        const uint32_t t_s = tmem + ((uint32_t)(32 * q) << 16);
        const uint32_t t_o = t_s + 64;
        const int out_row = ((row / a.wr) * a.W + row % a.wr) * a.C + h * 32;
        uint8_t *prow = sP + h * kTile + row * 128;
        uint32_t sph = 0, oph = 0;
        bool alive = true;
        for (int item = begin; item < end; ++item) {
            const int cb = item % a.ncb;
            const int br = item / a.ncb;
            const int r = br % a.R, b = br / a.R;
            const int32_t *routed = a.idx + (int64_t)br * a.topk;
            float m = -INFINITY, l = 0.f;
            float o[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = 0.f;
            int s_next = routed[0];
            for (int j = 0; j < a.topk; ++j) {
                const int s = s_next;
                if (j + 1 < a.topk) s_next = routed[j + 1];
                const bool ok = s >= 0 && s < a.R;
                if (alive) alive = mbar_wait(s_full, sph, a.err);
                sph ^= 1;
                tcgen05_after_sync();
                if (alive && ok) {
                    uint32_t v0[32], v1[32];
                    tmem_ld_32x32(t_s, v0);
                    tmem_ld_32x32(t_s + 32, v1);
                    tmem_wait_ld();
                    float mx = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(__uint_as_float(v0[c]), __uint_as_float(v1[c])));
                    const float mn = fmaxf(m, mx * a.scale_log2);
                    const float corr = fast_exp2(m - mn);
                    m = mn;
                    l *= corr;
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] *= corr;
                    // probabilities, packed to bf16 pairs and written as 8 swizzled 16-byte chunks
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = ch * 8 + 2 * e;
                            const float x0 = __uint_as_float(c < 32 ? v0[c] : v1[c - 32]);
                            const float x1 = __uint_as_float(c + 1 < 32 ? v0[c + 1] : v1[c + 1 - 32]);
                            const float p0 = bf16_trunc(fast_exp2(fmaf(x0, a.scale_log2, -mn)));
                            const float p1 = bf16_trunc(fast_exp2(fmaf(x1, a.scale_log2, -mn)));
                            l += p0 + p1;
                            w[e] = pack_bf16x2_trunc(p0, p1);
                        }
                        *reinterpret_cast<uint4 *>(prow + ((ch ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                fence_async_shared();
                tcgen05_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
                if (alive) alive = mbar_wait(o_full, oph, a.err);
                oph ^= 1;
                tcgen05_after_sync();
                if (alive && ok) {
                    uint32_t pv[32];
                    tmem_ld_32x32(t_o, pv);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] += __uint_as_float(pv[c]);
                }
                tcgen05_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free);
            }
            if (alive) {
                const float inv = l > 0.f ? __fdividef(1.f, l) : 0.f;
                const int qx = (r % a.n_win) * a.wr, qy = (r / a.n_win) * a.hr;
                __nv_bfloat16 *dst = a.out + (((int64_t)b * a.H + qy) * a.W + qx) * a.C + cb * 64 + out_row;
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    *reinterpret_cast<uint4 *>(dst + 8 * v) =
                        make_uint4(pack_bf16x2(o[8 * v] * inv, o[8 * v + 1] * inv),
                                   pack_bf16x2(o[8 * v + 2] * inv, o[8 * v + 3] * inv),
                                   pack_bf16x2(o[8 * v + 4] * inv, o[8 * v + 5] * inv),
                                   pack_bf16x2(o[8 * v + 6] * inv, o[8 * v + 7] * inv));
            }
        }
    }

    tcgen05_before_sync();
    __syncthreads();
    tcgen05_after_sync();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

bool gather_umma_supports(const Geometry &g)
{
    return g.hd == 32 && g.C % 64 == 0 && g.rs == 64 && g.wr <= 256 && g.hr <= 256 &&
           (long long)g.hr * g.W * g.C < (1LL << 31);
}

cudaError_t launch_attend_gather_umma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                      const int32_t *idx, void *out, const Geometry &g, int num_sms, unsigned *err,
                                      cudaStream_t stream)
{
    UmmaArgs a;
    a.idx = idx;
    a.err = err;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.H = g.H;
    a.W = g.W;
    a.C = g.C;
    a.n_win = g.n_win;
    a.topk = g.topk;
    a.R = g.R;
    a.hr = g.hr;
    a.wr = g.wr;
    a.ncb = g.C / 64;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    const long long nitems = (long long)g.B * g.R * a.ncb;
    if (nitems > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    a.nitems = (int)nitems;
    a.qslots = 2;
    a.kvslots = 2;
    a.idx_chunk = g.topk >= 32 ? 1 : 32 / g.topk;
    const size_t smem = 1024 + (size_t)kTile * (a.qslots + 2 * a.kvslots + 2) + 8 * (2 * a.qslots + 2 * a.kvslots + 5) +
                        4 * a.kvslots + 4 + 4 * (size_t)a.idx_chunk * g.topk;
    int grid = 2 * num_sms;
    if (grid > a.nitems) grid = a.nitems;
    a.per_cta = (a.nitems + grid - 1) / grid;
    grid = (a.nitems + a.per_cta - 1) / a.per_cta;
    static int granted[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)smem > granted[dev]) {
        e = cudaFuncSetAttribute(attend_gather_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        granted[dev] = (int)smem;
    }
    attend_gather_umma_kernel<<<grid, 192, smem, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace bra
