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
//    slots (128-byte swizzle, each CTA loading its own tiles), as in the mma.sync gather kernel;
//  * warp 1: allocates 256 TMEM columns (two S buffers at columns 0 and 64, two O buffers at
//    128 and 192); its lane 0 issues every MMA. Per routed region:
//      S_h = Q_h K_h^T  (M = 64 query rows, N = 64 keys, K = 32 channels of head h), head 0
//                        into TMEM lanes {0-15, 32-47, 64-79, 96-111}, head 1 into the same
//                        columns at lane offset 16 (an M = 64 accumulator fills 16 lanes of
//                        each 32-lane quadrant);
//      O = P V          (M = 128: the P rows of both heads, read from TMEM, N = 64 channels,
//                        K = 64 keys; V MN-major from shared memory); row p of O in TMEM lane
//                        p, of which the owner of that lane keeps its own head's 32 channels.
//    tcgen05.commit signals each product on an mbarrier and frees the query / KV slots.
//  * warps 2-5, softmax: thread t of warp w owns query row 16 (w % 4) + (t % 16) of head t / 16,
//    i.e. TMEM lane 32 (w % 4) + t. Per region it loads its 64 scores, updates the running max
//    and sum (exp2 with a log2(e) pre-scale; packed fp32 pairs), writes its 64 probabilities
//    rounded to bf16 as 32 pairs over the first 32 columns of its scores (P row = its TMEM
//    lane), then folds the region's PV product into 32 fp32 registers (o = o * correction +
//    PV). After the last region it normalises and stores its 32 output channels (64 bytes).
// Every wait is bounded (kErrTimeout); no thread leaves before the TMEM is released.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

constexpr int kRows = 64;                 // tokens per region = M of every MMA
constexpr int kTile = kRows * 128;        // 64 rows x 64 bf16 channels, 128-byte swizzled rows
constexpr uint32_t kTmemCols = 256;  // S buffers at 0 and 64, O buffers at 128 and 192
constexpr uint32_t kIdescS = umma_idesc_bf16(64, 64, false);  // Q K^T: B = K tile, K-major
constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 64, true);  // P V: A = both heads' P rows, B = V, MN-major

struct UmmaArgs {
    const int32_t *idx;
    unsigned *err;
    __nv_bfloat16 *out;
    int H, W, C, n_win, topk, R, hr, wr;  // H, W: the image in memory (the region grid may cover more)
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
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sKV + (size_t)a.kvslots * 2 * kTile);
    uint64_t *q_empty = q_full + a.qslots;
    uint64_t *kv_full = q_empty + a.qslots;
    uint64_t *kv_empty = kv_full + a.kvslots;
    uint64_t *s_full = kv_empty + a.kvslots;  // [2] per buffer
    uint64_t *p_full = s_full + 2;
    uint64_t *o_full = p_full + 2;
    uint64_t *o_free = o_full + 2;
    uint64_t *drain = o_free + 2;
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
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_free[i], 4);
        }
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
    grid_dependency_wait();  // the barriers and the TMEM are set up while the previous kernel drains

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
        // Units u = (item, routed region j) in CTA order. S(u) goes to TMEM buffer u & 1, where
        // the softmax overwrites its first 32 columns with P(u); PV(u - 1) follows once P(u - 1)
        // is written and the softmax has loaded O(u - 3). S(u) is issued after PV(u - 2), which
        // read the P that S(u) overwrites: the MMAs of this thread run in issue order. So
        // S(u + 1) and PV(u - 1) run while the softmax works on unit u.
        if (lane == 0) {
            const int units = (end - begin) * a.topk;
            int qs = 0;
            uint32_t qph = 0;
            bool alive = true, ok_prev = false;
            int kvs_prev = 0;
            // Descriptors of the tile bases; an offset of x bytes inside a tile is + (x >> 4).
            const uint64_t dq0 = umma_desc_sw128(smem_u32(sQ));
            const uint64_t dkv0 = umma_desc_sw128(smem_u32(sKV));
            constexpr uint64_t kTileStep = kTile >> 4;
            uint64_t dq = dq0;
            for (int u = 0; u <= units && alive; ++u) {
                bool ok = false;
                const int kvs = u % a.kvslots;
                if (u < units) {
                    const int j = u % a.topk;
                    if (j == 0) {
                        if (!(alive = mbar_wait(&q_full[qs], qph, a.err))) break;
                        dq = dq0 + (uint64_t)qs * kTileStep;
                    }
                    if (!(alive = mbar_wait(&kv_full[kvs], (uint32_t)((u / a.kvslots) & 1), a.err))) break;
                    const int b = u & 1;
                    tcgen05_after_sync();
                    ok = kv_ok[kvs] != 0;
                    if (ok) {
                        const uint64_t dk = dkv0 + (uint64_t)(2 * kvs) * kTileStep;
                        const uint32_t ds = tmem + 64 * b;
                        // S_h = Q_h K_h^T: head h's 32 channels start 64 h bytes into each row
                        umma_bf16(ds, dq + 0, dk + 0, kIdescS, 0u);
                        umma_bf16(ds, dq + 2, dk + 2, kIdescS, 1u);
                        umma_bf16(ds + (16u << 16), dq + 4, dk + 4, kIdescS, 0u);
                        umma_bf16(ds + (16u << 16), dq + 6, dk + 6, kIdescS, 1u);
                        umma_commit(&s_full[b]);
                    } else {
                        mbar_arrive(&s_full[b]);
                    }
                    if (j == a.topk - 1) {
                        umma_commit(&q_empty[qs]);
                        if (++qs == a.qslots) {
                            qs = 0;
                            qph ^= 1;
                        }
                    }
                }
                if (u >= 1) {
                    const int v = u - 1, bv = v & 1;
                    if (!(alive = mbar_wait(&p_full[bv], (uint32_t)((v >> 1) & 1), a.err))) break;
                    if (v >= 2 && !(alive = mbar_wait(&o_free[bv], (uint32_t)(((v >> 1) & 1) ^ 1), a.err))) break;
                    tcgen05_after_sync();
                    if (ok_prev) {
                        const uint64_t dv = dkv0 + (uint64_t)(2 * kvs_prev + 1) * kTileStep;
                        const uint32_t pa = tmem + 64 * bv;
                        const uint32_t d0 = tmem + 128 + 64 * bv;
                        // O = P V: A = the 128 P rows of both heads in TMEM (K = 64 keys, 8
                        // columns per 16-key step), B = all 64 channels of V (MN-major; the next
                        // 16 keys are 16 rows = 2048 bytes on). Row p of O lands in TMEM lane p;
                        // its thread keeps the 32 channels of its own head.
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16_ts(d0, pa + 8 * kk, dv + 128 * kk, kIdescPV, (uint32_t)kk);
                        umma_commit(&o_full[bv]);
                    } else {
                        mbar_arrive(&o_full[bv]);
                    }
                    umma_commit(&kv_empty[kvs_prev]);
                }
                ok_prev = ok;
                kvs_prev = kvs;
            }
            // every commit above arrives once the MMAs before it are done; wait for the last
            // one so that no arrival lands after this CTA has left
            umma_commit(drain);
            mbar_wait(drain, 0, a.err);
        }
    } else {
        // ------------------------------------------------------------- softmax warpgroup
        // Per unit u: load S(u), update the running max / sum of its item, write P(u); then fold
        // in PV(u - 1): added to the accumulator (kept relative to the max of the previous
        // unit) when it belongs to the same item, else it completes the previous item, which
        // is normalised and stored.
        const int q = warp & 3;  // the TMEM lane quadrant this warp may access
        const int h = lane >> 4;
        const int row = 16 * q + (lane & 15);
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int out_row = ((row / a.wr) * a.W + row % a.wr) * a.C + h * 32;
        const int units = (end - begin) * a.topk;
        bool alive = true, ok_prev = false;
        float m = -INFINITY, l = 0.f, l_prev = 0.f, corr = 1.f;
        float o[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0.f;
        __nv_bfloat16 *dst = nullptr, *dst_prev = nullptr;
        bool dst_in = false, dst_prev_in = false;  // the row's token lies inside the image
        // Routing indices run three units ahead of use, loaded with a volatile load at a fixed
        // place in the loop: the L2 latency under full HBM load is close to a microsecond.
        // (pb, pc, pj) = (image * R + region, channel block, routed slot) of the next load.
        int pb = begin / a.ncb, pc = begin % a.ncb, pj = 0;
        int sq[3] = {0, 0, 0};
        auto next_index = [&](int uu) -> int {
            int v = 0;
            if (uu < units) {
                v = ld_nc_volatile(a.idx + (int64_t)pb * a.topk + pj);
                if (++pj == a.topk) {
                    pj = 0;
                    if (++pc == a.ncb) {
                        pc = 0;
                        ++pb;
                    }
                }
            }
            return v;
        };
#pragma unroll
        for (int i = 0; i < 3; ++i) sq[i] = next_index(i);
        // ib, ic: image and channel block of the next item; rx, ry: column and row of its region
        const int ir = (begin / a.ncb) % a.R;
        int ic = begin % a.ncb, ib = (begin / a.ncb) / a.R;
        int rx = ir % a.n_win, ry = ir / a.n_win;
        int j = 0;  // routed slot of unit u
        bool start_prev = false;  // unit u - 1 opened its item
        for (int u = 0; u <= units; ++u) {
            bool ok = false;
            bool item_start = false;
            const float corr_prev = corr;  // max correction of unit u - 1
            if (u < units) {
                const int s = sq[0];
                sq[0] = sq[1];
                sq[1] = sq[2];
                sq[2] = next_index(u + 3);
                ok = s >= 0 && s < a.R;
                if (j == 0) {
                    item_start = true;
                    dst_prev = dst;
                    dst_prev_in = dst_in;
                    dst = a.out + (((int64_t)ib * a.H + ry * a.hr) * a.W + rx * a.wr) * a.C + ic * 64 + out_row;
                    dst_in = ry * a.hr + row / a.wr < a.H && rx * a.wr + row % a.wr < a.W;
                    if (++ic == a.ncb) {
                        ic = 0;
                        if (++rx == a.n_win) {
                            rx = 0;
                            if (++ry == a.n_win) {
                                ry = 0;
                                ++ib;
                            }
                        }
                    }
                    l_prev = l;
                    m = -INFINITY;
                    l = 0.f;
                }
                if (++j == a.topk) j = 0;
                const int b = u & 1;
                if (alive) alive = mbar_wait(&s_full[b], (uint32_t)((u >> 1) & 1), a.err);
                tcgen05_after_sync();
                corr = 1.f;
                if (alive && ok) {
                    uint32_t v0[32], v1[32];
                    tmem_ld_32x32(t_lane + 64 * b, v0);
                    tmem_ld_32x32(t_lane + 64 * b + 32, v1);
                    tmem_wait_ld();
                    // row max: four chains of three-input max
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(v0[c]), __uint_as_float(v0[c + 1]));
                        mx4[((c >> 1) + 2) & 3] =
                            fmax3(mx4[((c >> 1) + 2) & 3], __uint_as_float(v1[c]), __uint_as_float(v1[c + 1]));
                    }
                    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                    const float mn = fmaxf(m, mx * a.scale_log2);
                    corr = fast_exp2(m - mn);
                    m = mn;
                    // P row 32 q + lane (this thread's TMEM lane) over the first 32 columns of
                    // S: column j holds keys 2 j, 2 j + 1 rounded to bf16; the row sum is taken
                    // over the fp32 probabilities. Scale-and-shift, sums: packed fp32 pairs.
                    const float2 sc = make_float2(a.scale_log2, a.scale_log2), nm = make_float2(-mn, -mn);
                    float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                    make_float2(0.f, 0.f)};
                    uint32_t pw[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float x0 = __uint_as_float(j < 16 ? v0[2 * j] : v1[2 * j - 32]);
                        const float x1 = __uint_as_float(j < 16 ? v0[2 * j + 1] : v1[2 * j + 1 - 32]);
                        const float2 t = __ffma2_rn(make_float2(x0, x1), sc, nm);
                        const float2 pr = make_float2(fast_exp2(t.x), fast_exp2(t.y));
                        ls[j & 3] = __fadd2_rn(ls[j & 3], pr);
                        pw[j] = pack_bf16x2(pr.x, pr.y);
                    }
                    tmem_st_32x32(t_lane + 64 * b, pw);
                    tmem_wait_st();
                    const float2 lsum = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
                    l = l * corr + (lsum.x + lsum.y);
                }
                tcgen05_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[b]);
            }
            if (u >= 1) {
                const int v = u - 1, bv = v & 1;
                if (alive) alive = mbar_wait(&o_full[bv], (uint32_t)((v >> 1) & 1), a.err);
                tcgen05_after_sync();
                if (alive && ok_prev) {
                    // this thread's 32 output channels: columns 32 h of its O row (the column
                    // address of a TMEM load is the same for the whole warp, so both halves).
                    // The accumulator holds the item's earlier units relative to the max before
                    // unit v: o = o * corr(v) + PV(v), or o = PV(v) when v opened the item.
                    uint32_t w0[32], w1[32];
                    tmem_ld_32x32(t_lane + 128 + 64 * bv, w0);
                    tmem_ld_32x32(t_lane + 128 + 64 * bv + 32, w1);
                    tmem_wait_ld();
                    if (start_prev) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(h ? w1[c] : w0[c]);
                    } else {
                        const float2 cv = make_float2(corr_prev, corr_prev);
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const float2 r = __ffma2_rn(make_float2(o[c], o[c + 1]), cv,
                                                        make_float2(__uint_as_float(h ? w1[c] : w0[c]),
                                                                    __uint_as_float(h ? w1[c + 1] : w0[c + 1])));
                            o[c] = r.x;
                            o[c + 1] = r.y;
                        }
                    }
                } else if (start_prev) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = 0.f;  // a skipped first unit adds nothing
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] *= corr_prev;
                }
                tcgen05_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_free[bv]);
                if (u == units || item_start) {
                    // PV(u - 1) was the last region of the previous item: normalise and store it
                    const float lf = (u == units) ? l : l_prev;
                    __nv_bfloat16 *out = (u == units) ? dst : dst_prev;
                    const bool in_image = (u == units) ? dst_in : dst_prev_in;
                    const float inv = lf > 0.f ? __fdividef(1.f, lf) : 0.f;
                    if (alive && in_image) {
                        const float2 iv = make_float2(inv, inv);
                        uint32_t pk[16];
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const float2 r = __fmul2_rn(make_float2(o[c], o[c + 1]), iv);
                            pk[c / 2] = pack_bf16x2(r.x, r.y);
                        }
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            *reinterpret_cast<uint4 *>(out + 8 * x) = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                    }
                }
            }
            start_prev = item_start;
            ok_prev = ok;
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
                                      const int32_t *idx, void *out, const Geometry &g, int H, int W, int num_sms,
                                      unsigned *err, cudaStream_t stream)
{
    UmmaArgs a;
    a.idx = idx;
    a.err = err;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.H = H;
    a.W = W;
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
    a.qslots = 3;
    a.kvslots = 5;
    a.idx_chunk = g.topk >= 32 ? 1 : 32 / g.topk;
    const size_t smem = 1024 + (size_t)kTile * (a.qslots + 2 * a.kvslots) + 8 * (2 * a.qslots + 2 * a.kvslots + 9) +
                        4 * a.kvslots + 4 + 4 * (size_t)a.idx_chunk * g.topk;
    int grid = persistent_grid(a.nitems, num_sms);
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
    return launch_pdl(attend_gather_umma_kernel, dim3(grid), dim3(192), smem, stream, tq, tk, tv, a);
}

}  // namespace bra
