// bra_attend_mma.cu -- token-to-token attention over the routed regions on tensor cores (bf16).
//
// What it computes ("从零构建BiFormer", §2.2 TokenAttention; "医学图像分割模块：BiFormer /
// 双层路由注意力", §五 steps ⑤-⑦): for every query token of region r and every head, softmax
// (scale head_dim^-1/2) over the tokens of the regions idx[b, r, 0..topk-1], then the weighted
// sum of their values. Accumulation, softmax and normalisation are fp32; P is rounded to bf16
// for the PV product; out is rounded to bf16.
//
// Two kernels, both with K/V staged in shared memory by TMA (cp.async.bulk.tensor, 128-byte
// swizzle, each CTA loading its own tiles) and the gathered K/V never written to HBM:
//
// * gather: one CTA per (image, query region, group of 64-channel blocks). The query tile and,
//   per routed region, its K and V tiles (rs tokens x 64 channels each) arrive by TMA on
//   mbarriers, up to four regions in flight. Each warp owns 16 query rows of one head and runs
//   S = Q K^T and O += P V with mma.sync m16n8k16, folding the softmax online (exp2 with a
//   log2(e) pre-scale, running max and sum in registers). The output tile is staged in the
//   query tile's shared memory and written back by one TMA store. Needs rs % 16 == 0, rs <= 64.
//
// * dense: for tiny regions (rs of 1 or 4 tokens, where a 16-row MMA tile spans several query
//   regions). One CTA per (image, 64-channel block, band of query rows) stages the whole
//   image's K and V once; every query row attends to every key of the image with weight
//   cnt[region(query), region(key)] = number of times the key's region occurs in the query
//   region's idx row (0 masks it). That is exactly the gather semantics, duplicates included:
//   softmax over a concatenated key list weights each distinct key by its multiplicity. The
//   weight enters as +log2(cnt) on the logit. Needs R <= 64 and H * W <= 256.
#include "bra_device.cuh"
#include "bra_launch.h"
#include "bra_routing.cuh"

namespace bra {

constexpr int kRowBytes = 128;  // one token's 64 bf16 channels

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device, size high-water mark): later calls, including those made during CUDA
// graph capture, issue no attribute call.
template <typename Kernel>
static cudaError_t ensure_smem_limit(Kernel kernel, size_t bytes, int (&granted)[64])
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

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Rescales the running output and sum of one row pair by corr0 (row g) and corr1 (row g+8).
__device__ __forceinline__ void rescale(float (&o)[4][4], float (&l)[2], float corr0, float corr1)
{
    l[0] *= corr0;
    l[1] *= corr1;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        o[nt][0] *= corr0;
        o[nt][1] *= corr0;
        o[nt][2] *= corr1;
        o[nt][3] *= corr1;
    }
}

__device__ __forceinline__ float quad_max(float x)
{
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ float quad_sum(float x)
{
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// O += P V for KSTEPS 16-key steps; P in the S accumulators sc (fp32, rounded to bf16 here),
// V tile at vtile (keys x 64 channels, swizzled), key offset key0, head hb of the block.
template <int KSTEPS>
__device__ __forceinline__ void pv_product(float (&o)[4][4], const float (*sc)[4], uint32_t vtile, int key0, int hb,
                                           int lane)
{
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
        pa[1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
        pa[2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
        pa[3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            const int row = key0 + kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            ldmatrix_x4_trans(vtile + sw128(row, hb * 4 + np * 2 + (lane >> 4)), b0, b1, b2, b3);
            mma_bf16_16816(o[2 * np], pa, b0, b1);
            mma_bf16_16816(o[2 * np + 1], pa, b2, b3);
        }
    }
}

// Writes this warp's normalised 16 x 32 output (rows row0.., head hb) into a swizzled tile.
__device__ __forceinline__ void stage_output(uint32_t tile, const float (&o)[4][4], const float (&l)[2], int row0,
                                             int hb, int lane)
{
    const float l0 = quad_sum(l[0]), l1 = quad_sum(l[1]);
    const float inv0 = l0 > 0.f ? __fdividef(1.f, l0) : 0.f, inv1 = l1 > 0.f ? __fdividef(1.f, l1) : 0.f;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        st_shared_u32(tile + sw128(row0 + g, hb * 4 + nt) + 4 * t, pack_bf16x2(o[nt][0] * inv0, o[nt][1] * inv0));
        st_shared_u32(tile + sw128(row0 + g + 8, hb * 4 + nt) + 4 * t, pack_bf16x2(o[nt][2] * inv1, o[nt][3] * inv1));
    }
}

struct GatherArgs {
    const int32_t *idx;
    unsigned *err;
    __nv_bfloat16 *out;   // [B, H, W, C]
    int H, W, C;          // the image in memory (the region grid may cover more)
    int n_win, topk, R, hr, wr;
    int ncb;          // 64-channel blocks in C
    int ncb_per_cta;  // channel blocks one work item covers (NCB)
    int groups;       // work items per (image, region)
    int nitems;       // B * R * groups
    int per_cta;      // contiguous work items per CTA
    int ncw;          // consumer warps = NCB * 2 heads * rs / 16 row tiles
    int qslots, kvslots, idx_chunk;
    int per_head;     // idx is [B, heads, R, topk]: every head gathers its own regions
    int heads;
    float scale_log2;
};

constexpr int kGatherMaxHeads = 8;  // heads of one work item (NCB <= 4 blocks of 2 heads)

// Per-lane byte offsets of the ldmatrix rows inside 128-byte-swizzled tiles. Every row a lane
// addresses has the same (row & 7), so the swizzle XOR depends on the lane only and the
// offsets of later 8-row groups are compile-time constants (+1024 per 8 rows).
struct LaneOffsets {
    uint32_t q[2];   // Q tile, 16-row tile rt, k-steps 0 and 1 of head hb
    uint32_t k;      // K tile, keys (lane & 7) + 8 nt, channels of head hb
    uint32_t v[2];   // V tile (transposed loads), keys + 16 kk, channel pairs np = 0, 1
};

__device__ __forceinline__ LaneOffsets lane_offsets(int rt, int hb, int lane)
{
    LaneOffsets o;
    const int x = lane & 7;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) o.q[ks] = sw128(rt * 16 + (lane & 15), hb * 4 + ks * 2 + (lane >> 4));
    o.k = (uint32_t)x * 128u + ((uint32_t)((hb * 4 + (lane >> 3)) ^ x) << 4);
#pragma unroll
    for (int np = 0; np < 2; ++np)
        o.v[np] = (uint32_t)(x + ((lane >> 3) & 1) * 8) * 128u + ((uint32_t)((hb * 4 + np * 2 + (lane >> 4)) ^ x) << 4);
    return o;
}

// S = Q K^T for one 16-row tile of one head against one routed region (NT 8-key n-tiles),
// online-softmax update of (m, l, o), then O += P V. P is rounded down to bf16 (the low
// half of the fp32 bits dropped) and the row sums accumulate exactly those values, so the
// normalisation matches the weights used.
template <int NT>
__device__ __forceinline__ void attend_region(float (&o)[4][4], float (&m)[2], float (&l)[2], const uint32_t (&qf)[2][4],
                                              uint32_t ktile, uint32_t vtile, const LaneOffsets &off, float scale_log2)
{
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(ktile + off.k + nt * 1024, b0, b1, b2, b3);
        mma_bf16_16816(sc[nt], qf[0], b0, b1);
        mma_bf16_16816(sc[nt], qf[1], b2, b3);
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
    }
    const float mn0 = fmaxf(m[0], quad_max(mx0) * scale_log2);
    const float mn1 = fmaxf(m[1], quad_max(mx1) * scale_log2);
    rescale(o, l, fast_exp2(m[0] - mn0), fast_exp2(m[1] - mn1));
    m[0] = mn0;
    m[1] = mn1;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = bf16_trunc(fast_exp2(fmaf(sc[nt][0], scale_log2, -mn0)));
        sc[nt][1] = bf16_trunc(fast_exp2(fmaf(sc[nt][1], scale_log2, -mn0)));
        sc[nt][2] = bf16_trunc(fast_exp2(fmaf(sc[nt][2], scale_log2, -mn1)));
        sc[nt][3] = bf16_trunc(fast_exp2(fmaf(sc[nt][3], scale_log2, -mn1)));
        l[0] += sc[nt][0] + sc[nt][1];
        l[1] += sc[nt][2] + sc[nt][3];
    }
#pragma unroll
    for (int kk = 0; kk < NT / 2; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2_trunc(sc[2 * kk][0], sc[2 * kk][1]);
        pa[1] = pack_bf16x2_trunc(sc[2 * kk][2], sc[2 * kk][3]);
        pa[2] = pack_bf16x2_trunc(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
        pa[3] = pack_bf16x2_trunc(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(vtile + off.v[np] + kk * 2048, b0, b1, b2, b3);
            mma_bf16_16816(o[2 * np], pa, b0, b1);
            mma_bf16_16816(o[2 * np + 1], pa, b2, b3);
        }
    }
}

// Item coordinates the producer publishes with each query slot: image, the query region's
// top-left token (x, y), first channel block and number of channel blocks.
struct ItemInfo {
    int b, qx, qy, cb;
};

// Persistent, warp-specialised gather attention. Each CTA owns a contiguous run of work
// items (image, query region, group of NCB 64-channel blocks), in image order.
//  * Warp `ncw` (producer): stages the idx rows of the next items in shared memory, then
//    one lane issues the TMA loads: the query tile into a ring of `qslots` slots and, per
//    routed region, its K and V tiles into a ring of `kvslots` slots; each slot has a
//    "full" mbarrier (TMA transaction bytes) and an "empty" one (one arrival per consumer
//    warp). An idx entry outside [0, R) fills its slot with nothing and is flagged.
//    Per-head routing (per_head): routed slot j of an item holds, for each of its 2 NCB heads,
//    the K and V tiles (one 64-channel block) of that head's own j-th region; the head's
//    warps read their 32 channels of it. (The other 32 channels of the tile are loaded too:
//    a 64-channel box keeps the 128-byte swizzled layout of the shared-index path.)
//  * Warps 0..ncw-1 (consumers): warp w owns 16 query rows (w % RT) of head (w / RT) % 2 of
//    channel block w / (2 RT); it runs attend_region per routed region, then writes its
//    normalised output into one of two output tiles; one thread stores the tile by TMA
//    while the next item is computed.
// Every wait is bounded; a wait that gives up flags kErrTimeout and the thread stops
// computing but keeps arriving on barriers, so the CTA still finishes.
template <int RS>
__global__ void __launch_bounds__(288, 2) attend_gather_mma_kernel(const __grid_constant__ CUtensorMap tq,
                                                                   const __grid_constant__ CUtensorMap tk,
                                                                   const __grid_constant__ CUtensorMap tv,
                                                                   const __grid_constant__ CUtensorMap tout,
                                                                   const GatherArgs a)
{
    constexpr int RT = RS / 16;           // 16-row tiles per region
    constexpr int NT = RS / 8;            // 8-key n-tiles per region
    constexpr int TILE = RS * kRowBytes;  // one (region, 64-channel block) tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NCB = a.ncb_per_cta;
    const int kv_tiles = (a.per_head ? 4 : 2) * NCB;  // tiles of one KV slot
    uint8_t *sQ = smem;
    uint8_t *sKV = sQ + (size_t)a.qslots * NCB * TILE;
    uint64_t *full_q = reinterpret_cast<uint64_t *>(sKV + (size_t)a.kvslots * kv_tiles * TILE);
    uint64_t *empty_q = full_q + a.qslots;
    uint64_t *full_kv = empty_q + a.qslots;
    uint64_t *empty_kv = full_kv + a.kvslots;
    int *kv_ok = reinterpret_cast<int *>(empty_kv + a.kvslots);  // [kvslots][kGatherMaxHeads]
    ItemInfo *qinfo = reinterpret_cast<ItemInfo *>(kv_ok + a.kvslots * kGatherMaxHeads);
    int *sidx = reinterpret_cast<int *>(qinfo + a.qslots);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int begin = blockIdx.x * a.per_cta;
    const int end = min(a.nitems, begin + a.per_cta);
    grid_dependency_wait();

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.qslots; ++i) {
            mbar_init(&full_q[i], 1);
            mbar_init(&empty_q[i], a.ncw);
        }
        for (int i = 0; i < a.kvslots; ++i) {
            mbar_init(&full_kv[i], 1);
            mbar_init(&empty_kv[i], a.ncw);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == a.ncw) {
        // ------------------------------------------------------------- producer warp
        int qs = 0, kvs = 0;
        uint32_t qph = 0, kvph = 0;
        bool alive = true;
        for (int c0 = begin; c0 < end; c0 += a.idx_chunk) {
            const int n = min(a.idx_chunk, end - c0);
            __syncwarp();
            // index rows of the chunk's items: one per item, or (per_head) one per head of it,
            // -2 for a head past C (nothing to load, nothing to flag)
            const int hpi = a.per_head ? 2 * NCB : 1;
            for (int e = lane; e < n * hpi * a.topk; e += 32) {
                const int il = e / (hpi * a.topk), rem = e - il * (hpi * a.topk);
                const int hh = rem / a.topk, j = rem - hh * a.topk;
                const int it = c0 + il;
                if (a.per_head) {
                    const int br = it / a.groups, grp = it - br * a.groups;
                    const int r = br % a.R, b = br / a.R, h = 2 * grp * NCB + hh;
                    sidx[e] = h < a.heads ? a.idx[(((int64_t)b * a.heads + h) * a.R + r) * a.topk + j] : -2;
                } else {
                    sidx[e] = a.idx[(int64_t)(it / a.groups) * a.topk + j];
                }
            }
            __syncwarp();
            if (lane != 0 || !alive) continue;
            for (int i = 0; i < n && alive; ++i) {
                const int item = c0 + i;
                const int grp = item % a.groups;
                const int br = item / a.groups;
                const int r = br % a.R, b = br / a.R;
                const int cb0 = grp * NCB, nh = min(NCB, a.ncb - cb0);
                const int qx = (r % a.n_win) * a.wr, qy = (r / a.n_win) * a.hr;
                if (!(alive = mbar_wait(&empty_q[qs], qph ^ 1, a.err))) break;
                qinfo[qs] = ItemInfo{b, qx, qy, (cb0 << 8) | nh};
                // one box brings all NCB channel-block tiles (blocks past C are zero-filled and
                // counted like the others)
                mbar_arrive_expect_tx(&full_q[qs], (uint32_t)(NCB * TILE));
                tma_load_5d(sQ + (size_t)qs * NCB * TILE, &tq, 0, qx, qy, cb0, b, &full_q[qs]);
                if (++qs == a.qslots) {
                    qs = 0;
                    qph ^= 1;
                }
                for (int j = 0; j < a.topk; ++j) {
                    if (!(alive = mbar_wait(&empty_kv[kvs], kvph ^ 1, a.err))) break;
                    if (a.per_head) {
                        // K tiles of the item's heads, then their V tiles (box: one block)
                        uint8_t *kt = sKV + (size_t)kvs * 4 * NCB * TILE;
                        int nload = 0;
                        for (int hh = 0; hh < hpi; ++hh) {
                            const int s = sidx[(i * hpi + hh) * a.topk + j];
                            const bool ok = s >= 0 && s < a.R;
                            if (!ok && s != -2) flag_error(a.err, kErrIndex);
                            kv_ok[kvs * kGatherMaxHeads + hh] = ok;
                            nload += ok ? 1 : 0;
                        }
                        mbar_arrive_expect_tx(&full_kv[kvs], (uint32_t)(2 * nload * TILE));
                        for (int hh = 0; hh < hpi; ++hh) {
                            const int s = sidx[(i * hpi + hh) * a.topk + j];
                            if (s < 0 || s >= a.R) continue;
                            const int sx = (s % a.n_win) * a.wr, sy = (s / a.n_win) * a.hr;
                            tma_load_5d(kt + (size_t)hh * TILE, &tk, 0, sx, sy, cb0 + hh / 2, b, &full_kv[kvs]);
                            tma_load_5d(kt + (size_t)(2 * NCB + hh) * TILE, &tv, 0, sx, sy, cb0 + hh / 2, b,
                                        &full_kv[kvs]);
                        }
                    } else {
                        const int s = sidx[i * a.topk + j];
                        const bool ok = s >= 0 && s < a.R;
                        kv_ok[kvs * kGatherMaxHeads] = ok;
                        if (ok) {
                            const int sx = (s % a.n_win) * a.wr, sy = (s / a.n_win) * a.hr;
                            mbar_arrive_expect_tx(&full_kv[kvs], (uint32_t)(2 * NCB * TILE));
                            uint8_t *kt = sKV + (size_t)kvs * 2 * NCB * TILE;
                            tma_load_5d(kt, &tk, 0, sx, sy, cb0, b, &full_kv[kvs]);
                            tma_load_5d(kt + NCB * TILE, &tv, 0, sx, sy, cb0, b, &full_kv[kvs]);
                        } else {
                            flag_error(a.err, kErrIndex);
                            mbar_arrive_expect_tx(&full_kv[kvs], 0);
                        }
                    }
                    if (++kvs == a.kvslots) {
                        kvs = 0;
                        kvph ^= 1;
                    }
                }
            }
        }
        return;
    }

    // ----------------------------------------------------------------- consumer warps
    const int rt = warp % RT, hb = (warp / RT) & 1, cbl = warp / (2 * RT);
    const LaneOffsets off = lane_offsets(rt, hb, lane);
    // this warp's K tile in a KV slot, the distance from it to its V tile, its validity flag
    const int kt_index = a.per_head ? cbl * 2 + hb : cbl;
    const int v_dist = a.per_head ? 2 * NCB : NCB;
    const int ok_index = a.per_head ? cbl * 2 + hb : 0;
    // element offsets, inside the region's first token, of this lane's two output rows
    // (rows g and g + 8 of the 16-row tile), channel pair 2t of head hb
    int row_off[2], row_y[2], row_x[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int ri = rt * 16 + (lane >> 2) + 8 * h;
        row_y[h] = ri / a.wr;
        row_x[h] = ri % a.wr;
        row_off[h] = (row_y[h] * a.W + row_x[h]) * a.C + hb * 32 + 2 * (lane & 3);
    }
    int qs = 0, kvs = 0;
    uint32_t qph = 0, kvph = 0;
    bool alive = true;
    for (int item = begin; item < end; ++item) {
        uint32_t qf[2][4];
        if (alive) alive = mbar_wait(&full_q[qs], qph, a.err);
        const ItemInfo info = qinfo[qs];
        const int cb0 = info.cb >> 8, nh = info.cb & 0xff;
        const bool active = cbl < nh;
        if (alive && active) {
            const uint32_t qtile = smem_u32(sQ + (size_t)(qs * NCB + cbl) * TILE);
            ldmatrix_x4(qtile + off.q[0], qf[0][0], qf[0][1], qf[0][2], qf[0][3]);
            ldmatrix_x4(qtile + off.q[1], qf[1][0], qf[1][1], qf[1][2], qf[1][3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_q[qs]);
        if (++qs == a.qslots) {
            qs = 0;
            qph ^= 1;
        }

        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
        float o[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        for (int j = 0; j < a.topk; ++j) {
            if (alive) alive = mbar_wait(&full_kv[kvs], kvph, a.err);
            if (alive && active && kv_ok[kvs * kGatherMaxHeads + ok_index]) {
                const uint32_t ktile = smem_u32(sKV + (size_t)(kvs * kv_tiles + kt_index) * TILE);
                attend_region<NT>(o, m, l, qf, ktile, ktile + v_dist * TILE, off, a.scale_log2);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_kv[kvs]);
            if (++kvs == a.kvslots) {
                kvs = 0;
                kvph ^= 1;
            }
        }

        // epilogue: normalise and store this warp's 16 x 32 output straight to global memory
        if (alive && active) {
            const float l0 = quad_sum(l[0]), l1 = quad_sum(l[1]);
            const float inv0 = l0 > 0.f ? __fdividef(1.f, l0) : 0.f, inv1 = l1 > 0.f ? __fdividef(1.f, l1) : 0.f;
            __nv_bfloat16 *dst = a.out + (((int64_t)info.b * a.H + info.qy) * a.W + info.qx) * a.C + (cb0 + cbl) * 64;
            // rows of a padded map outside the image are not stored
            const bool in0 = info.qy + row_y[0] < a.H && info.qx + row_x[0] < a.W;
            const bool in1 = info.qy + row_y[1] < a.H && info.qx + row_x[1] < a.W;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                if (in0)
                    *reinterpret_cast<uint32_t *>(dst + row_off[0] + nt * 8) = pack_bf16x2(o[nt][0] * inv0, o[nt][1] * inv0);
                if (in1)
                    *reinterpret_cast<uint32_t *>(dst + row_off[1] + nt * 8) = pack_bf16x2(o[nt][2] * inv1, o[nt][3] * inv1);
            }
        }
    }
}

bool gather_mma_supports(const Geometry &g)
{
    return g.hd == 32 && g.C % 64 == 0 && g.rs % 16 == 0 && g.rs <= 64 && g.wr <= 256 && g.hr <= 256 &&
           (long long)g.hr * g.W * g.C < (1LL << 31);
}

// 64-channel blocks per work item: eight consumer warps of 16 rows x 1 head at most.
static int gather_blocks_per_item(const Geometry &g)
{
    const int rt = g.rs / 16;
    int n = 8 / (2 * rt);
    if (n < 1) n = 1;
    if (n > g.C / 64) n = g.C / 64;
    return n;
}

void gather_mma_box(const Geometry &g, int box[5])
{
    box[0] = 64;
    box[1] = g.wr;
    box[2] = g.hr;
    box[3] = gather_blocks_per_item(g);
    box[4] = 1;
}

template <int RS>
static cudaError_t launch_gather_rs(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                    const CUtensorMap &tout, const GatherArgs &a, int grid, size_t smem,
                                    cudaStream_t stream)
{
    static_assert(RS % 16 == 0 && RS <= 64, "tokens per region");
    static int granted[64] = {0};
    cudaError_t e = ensure_smem_limit(attend_gather_mma_kernel<RS>, smem, granted);
    if (e != cudaSuccess) return e;
    return launch_pdl(attend_gather_mma_kernel<RS>, dim3(grid), dim3((a.ncw + 1) * 32), smem, stream, tq, tk, tv, tout,
                      a);
}

cudaError_t launch_attend_gather_mma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                     const CUtensorMap &tout, const int32_t *idx, void *out, const Geometry &g, int H,
                                     int W, int num_sms, unsigned *err, cudaStream_t stream, bool per_head)
{
    GatherArgs a;
    a.per_head = per_head ? 1 : 0;
    a.heads = g.heads;
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
    const int rt = g.rs / 16;
    const int ncb_per_cta = gather_blocks_per_item(g);
    a.ncb_per_cta = ncb_per_cta;
    a.groups = (a.ncb + ncb_per_cta - 1) / ncb_per_cta;
    a.ncw = ncb_per_cta * 2 * rt;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    const long long nitems = (long long)g.B * g.R * a.groups;
    if (nitems > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    a.nitems = (int)nitems;
    // Two CTAs per SM with ~111 KB of shared memory each for the rings; for regions of 16 tokens
    // (one 16-row tile per head, at most 160 threads at 88 registers) four CTAs per SM with
    // ~52 KB each: the consumer warps' per-item chains are short, so more of them in flight pay
    // more than deeper rings (stage2: 32.5 -> 26.6 us).
    const int per_sm = (g.rs <= 16 && a.ncw <= 4) ? 4 : 2;
    const size_t tile = (size_t)g.rs * kRowBytes * ncb_per_cta;  // one slot of one tensor
    const size_t kv_tile = (per_head ? 4 : 2) * tile;                // one KV slot
    const size_t budget = (per_sm == 4 ? 52 : 111) * 1024;
    a.qslots = per_head ? 2 : (g.topk <= 2 ? 4 : 2);
    long long kv = (long long)((budget - a.qslots * tile) / kv_tile);
    if (kv > 8) kv = 8;
    if (kv < 2) kv = 2;
    a.kvslots = (int)kv;
    a.idx_chunk = g.topk >= 32 ? 1 : 32 / g.topk;
    const int hpi = per_head ? 2 * ncb_per_cta : 1;  // index rows per item
    const size_t smem = 1024 + tile * a.qslots + kv_tile * a.kvslots + 16 * (a.qslots + a.kvslots) +
                        4 * (size_t)kGatherMaxHeads * a.kvslots + sizeof(ItemInfo) * a.qslots +
                        4 * (size_t)a.idx_chunk * g.topk * hpi;
    int grid = persistent_grid(a.nitems, num_sms, per_sm);
    a.per_cta = (a.nitems + grid - 1) / grid;
    grid = (a.nitems + a.per_cta - 1) / a.per_cta;
    switch (g.rs) {
    case 16: return launch_gather_rs<16>(tq, tk, tv, tout, a, grid, smem, stream);
    case 32: return launch_gather_rs<32>(tq, tk, tv, tout, a, grid, smem, stream);
    case 48: return launch_gather_rs<48>(tq, tk, tv, tout, a, grid, smem, stream);
    case 64: return launch_gather_rs<64>(tq, tk, tv, tout, a, grid, smem, stream);
    default: return cudaErrorInvalidValue;
    }
}

// ------------------------------------------------------------------------- dense kernel

struct DenseArgs {
    const int32_t *idx;
    int32_t *idx_out;  // ROUTE: the index this kernel selects, [B, R, topk]
    unsigned *err;
    int H, W, n_win, topk, R, hr, wr, N, npad;
    int ncb;             // 64-channel blocks in C
    int cpb;             // 64-channel blocks per CTA
    int rows_per_split;  // image rows of queries per CTA
    int nsplit;
    float scale_log2;
    float route_scale;  // ROUTE: C^-1/2
    int inputs_ready;   // q, k, v may be loaded before the wait for the previous kernel
    int Hm;             // image rows in memory (H: the region grid's, which may be more)
    int per_head;       // idx is [B, heads, R, topk]: each head of the block has its own counts
    int heads;
};

constexpr int kDensePartPad = 68;  // row stride (floats) of a partial affinity tile
constexpr int kDenseMaxBlocks = 16;  // 64-channel blocks of an image the fused routing adds (C <= 1024)

// The routing step of one-token regions inside the dense kernel (ROUTE), for a cluster of CTAs
// that together hold one image's q and k, each CTA `cpb` 64-channel blocks of it:
//  1. each CTA forms, per block, the 64 x 64 tile of partial dot products q_i . k_s over the
//     block's channels with the MMA sequence of route_tokens_mma_kernel (two 32-channel chunks
//     in order, 8 channels per lane), so every partial is the same bits as that kernel's partial
//     of the block;
//  2. after a cluster barrier, CTA `ct` takes rows ct, ct + nct, ...: for each (row, region) it
//     adds the partials of blocks 0, 1, ... in order from the CTAs' shared memory (distributed
//     shared memory, plain loads), scales by C^-1/2 and forms the routing key; the keys of a row
//     are distinct, so the position of region s in the row's descending order is the number of
//     keys above its own, which one thread per (row, region) counts. A region whose position is
//     below topk is written there in the index, and cnt[row][s] = 1 is set in every CTA of the
//     cluster (the selected regions of a row are distinct). This is the order the routing
//     kernel's sort gives, so the index is the same bits;
//  3. a second cluster barrier publishes cnt, and no CTA touches another's memory after it.
__device__ __forceinline__ void dense_route_rows(const DenseArgs &a, const float *part, int *cnt,
                                                 unsigned long long *skey, int b, int ct, int nct)
{
    const uint32_t part0 = smem_u32(part);
    const int nrows = (a.R - ct + nct - 1) / nct;  // rows ct, ct + nct, ... below R
    const int cshift = a.cpb == 2 ? 1 : 0;          // block w sits in CTA w >> cshift
    // (row, region) pairs as rr * 64 + s (shifts, no division); regions s >= R are skipped
    for (int e = threadIdx.x; e < nrows * 64; e += blockDim.x) {
        const int rr = e >> 6, s = e & 63;
        if (s >= a.R) continue;
        const int i = ct + nct * rr;
        const uint32_t base = part0 + 4u * (uint32_t)(i * kDensePartPad + s);
        // every block's partial in flight at once, then added in block order
        float pw[kDenseMaxBlocks];
#pragma unroll
        for (int w = 0; w < kDenseMaxBlocks; ++w)
            pw[w] = w < a.ncb ? ld_cluster_f32(cluster_map(base + 4u * (uint32_t)((w & (a.cpb - 1)) * 64 * kDensePartPad),
                                                            (uint32_t)(w >> cshift)))
                              : 0.f;
        float d = 0.f;
#pragma unroll
        for (int w = 0; w < kDenseMaxBlocks; ++w)
            if (w < a.ncb) d += pw[w];
        skey[rr * 64 + s] = routing_key(d * a.route_scale, s);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nrows * 64; e += blockDim.x) {
        const int rr = e >> 6, s = e & 63;
        if (s >= a.R) continue;
        const unsigned long long *row = skey + rr * 64;
        const unsigned long long mine = row[s];
        int pos = 0;
#pragma unroll 7
        for (int j = 0; j < a.R; ++j) pos += row[j] > mine ? 1 : 0;
        if (pos < a.topk) {
            const int i = ct + nct * rr;
            a.idx_out[((int64_t)b * a.R + i) * a.topk + pos] = s;
            const uint32_t at = smem_u32(cnt + i * a.R + s);
            for (int r = 0; r < nct; ++r) st_cluster_u32(cluster_map(at, (uint32_t)r), 1u);
        }
    }
}

// MIN_CTAS: CTAs per SM the registers are budgeted for (2, or 3 when three CTAs' shared memory
// fits on an SM). ROUTE: one-token regions, the kernel selects the index itself (launched as a
// cluster of the CTAs of one image; above).
template <int MIN_CTAS, bool ROUTE>
__global__ void __launch_bounds__(256, MIN_CTAS) attend_dense_mma_kernel(const __grid_constant__ CUtensorMap tq,
                                                               const __grid_constant__ CUtensorMap tk,
                                                               const __grid_constant__ CUtensorMap tv,
                                                               const __grid_constant__ CUtensorMap tout,
                                                               const DenseArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nq = a.rows_per_split * a.W;  // query rows of this CTA (the last split may run past H)
    const int nqpad = (nq + 15) & ~15;
    const int cpb = a.cpb;
    const size_t qtile = (size_t)nqpad * kRowBytes, kvtile = (size_t)a.npad * kRowBytes;
    uint8_t *sQ = smem;               // [cpb] x [nqpad rows]
    uint8_t *sK = sQ + cpb * qtile;   // [cpb] x [npad rows]
    uint8_t *sV = sK + cpb * kvtile;  // [cpb] x [npad rows]
    const int nct = a.ncb / cpb;  // CTAs per (image, band of rows); ROUTE: the cluster
    // ROUTE: [cpb][64][kDensePartPad] partial affinities, then the routing keys of this CTA's
    // rows, [ceil(R / nct)][64]
    float *part = reinterpret_cast<float *>(sV + cpb * kvtile);
    unsigned long long *skey =
        reinterpret_cast<unsigned long long *>(part + (ROUTE ? cpb * 64 * kDensePartPad : 0));
    // [planes][R][R]: the multiplicity of each (query region, key region) pair, then, in place,
    // its log2; one plane, or (per-head routing) one per head of the block
    const int planes = a.per_head ? 2 : 1;
    int *cnt = reinterpret_cast<int *>(skey + (ROUTE ? ((a.R + nct - 1) / nct) * 64 : 0));
    float *lw = reinterpret_cast<float *>(cnt);
    uint8_t *reg = reinterpret_cast<uint8_t *>(cnt + planes * a.R * a.R);  // [npad] region of each key
    uint64_t *bar = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(reg + a.npad) + 7) & ~uintptr_t(7));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    int64_t item = blockIdx.x;
    const int split = (int)(item % a.nsplit);
    item /= a.nsplit;
    const int ct = (int)(item % nct);
    const int b = (int)(item / nct);
    const int cb0 = ct * cpb;
    const int y0 = split * a.rows_per_split;

    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    // q, k and v: before the wait for the previous kernel when that kernel is the routing step of
    // the same forward pass (it already waited for their producers), else after it
    if (!a.inputs_ready) grid_dependency_wait();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(cpb * (nq + 2 * a.N) * kRowBytes));
        for (int j = 0; j < cpb; ++j) {
            tma_load_4d(sQ + j * qtile, &tq, (cb0 + j) * 64, 0, y0, b, bar);
            tma_load_4d(sK + j * kvtile, &tk, (cb0 + j) * 64, 0, 0, b, bar);
            tma_load_4d(sV + j * kvtile, &tv, (cb0 + j) * 64, 0, 0, b, bar);
        }
    }
    // zero the padding rows (TMA writes rows [0, nq) and [0, N) only)
    for (int j = 0; j < cpb; ++j) {
        for (int i = threadIdx.x; i < (nqpad - nq) * 8; i += blockDim.x)
            reinterpret_cast<uint4 *>(sQ + j * qtile + (size_t)nq * kRowBytes)[i] = make_uint4(0, 0, 0, 0);
        for (int i = threadIdx.x; i < (a.npad - a.N) * 8; i += blockDim.x) {
            reinterpret_cast<uint4 *>(sK + j * kvtile + (size_t)a.N * kRowBytes)[i] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4 *>(sV + j * kvtile + (size_t)a.N * kRowBytes)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    for (int t = threadIdx.x; t < a.npad; t += blockDim.x)
        reg[t] = t < a.N ? (uint8_t)(((t / a.W) / a.hr) * a.n_win + (t % a.W) / a.wr) : 0;
    for (int e = threadIdx.x; e < planes * a.R * a.R; e += blockDim.x) cnt[e] = 0;
    bool alive = true;
    if constexpr (ROUTE) {
        // the partial affinities of this CTA's blocks: task = (block j, 16-row tile, key half)
        __syncthreads();
        alive = mbar_wait(bar, 0, a.err);
        const int g = lane >> 2, c = lane & 3;
        const int rtn = (a.R + 15) >> 4, ntiles = (a.R + 7) >> 3;
        for (int task = warp; task < cpb * 8; task += nwarps) {
            const int j = task >> 3, rt = (task >> 1) & 3, half = task & 1;
            if (rt >= rtn) continue;
            const uint8_t *qt = sQ + j * qtile, *kt = sK + j * kvtile;
            float acc[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const uint4 xa = *reinterpret_cast<const uint4 *>(qt + sw128(16 * rt + g, 4 * ch + c));
                const uint4 xb = *reinterpret_cast<const uint4 *>(qt + sw128(16 * rt + g + 8, 4 * ch + c));
                const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};
                const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int nt = 4 * half + n;
                    if (nt < ntiles) {
                        const uint4 y = *reinterpret_cast<const uint4 *>(kt + sw128(8 * nt + g, 4 * ch + c));
                        mma_bf16_16816(acc[n], a0, y.x, y.y);
                        mma_bf16_16816(acc[n], a1, y.z, y.w);
                    }
                }
            }
            float *pj = part + (size_t)j * 64 * kDensePartPad;
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int nt = 4 * half + n;
                if (nt < ntiles) {
                    *reinterpret_cast<float2 *>(pj + (16 * rt + g) * kDensePartPad + 8 * nt + 2 * c) =
                        make_float2(acc[n][0], acc[n][1]);
                    *reinterpret_cast<float2 *>(pj + (16 * rt + g + 8) * kDensePartPad + 8 * nt + 2 * c) =
                        make_float2(acc[n][2], acc[n][3]);
                }
            }
        }
        cluster_sync();  // every CTA's partials and zeroed cnt, before any remote access
        dense_route_rows(a, part, cnt, skey, b, ct, nct);
        cluster_sync();  // cnt complete in every CTA; no remote access after this point
    } else {
        if (a.inputs_ready) grid_dependency_wait();  // idx comes from the previous kernel
        __syncthreads();
        // multiplicity of every routed region: the image's idx entries (per-head routing: the rows
        // of this block's two heads, one plane each), eight loads per thread in flight at once,
        // then one shared-memory count per entry
        const int32_t *routed = a.per_head ? a.idx + ((int64_t)b * a.heads + 2 * cb0) * a.R * a.topk
                                           : a.idx + (int64_t)b * a.R * a.topk;
        const int nent = planes * a.R * a.topk;  // a plane's rows follow the previous plane's
        const bool flagger = split == 0 && (a.per_head || ct == 0);
        for (int e0 = threadIdx.x; e0 < nent; e0 += 8 * blockDim.x) {
            int sv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * blockDim.x;
                sv[u] = e < nent ? routed[e] : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * blockDim.x;
                if (e < nent) {
                    const int s = sv[u];
                    if (s >= 0 && s < a.R)
                        atomicAdd(&cnt[(e / a.topk) * a.R + s], 1);  // row e / topk of plane-major rows
                    else if (flagger)
                        flag_error(a.err, kErrIndex);
                }
            }
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < planes * a.R * a.R; e += blockDim.x) {
        const int c = cnt[e];
        lw[e] = c == 1 ? 0.f : (c ? log2f((float)c) : -INFINITY);  // log2(1) = 0 exactly: skip the call
    }
    __syncthreads();

    if constexpr (!ROUTE) alive = mbar_wait(bar, 0, a.err);
    const int g = lane >> 2, t = lane & 3;
    const int tasks = (nqpad / 16) * 2 * cpb;  // (16-row tile, block, head of the block)

    for (int task = warp; alive && task < tasks; task += nwarps) {
        const int rt = task / (2 * cpb), rem = task - rt * 2 * cpb;
        const int j = rem >> 1, hb = rem & 1;
        const uint32_t qbase = smem_u32(sQ + j * qtile), kbase = smem_u32(sK + j * kvtile);
        const uint32_t vbase = smem_u32(sV + j * kvtile);
        uint32_t qf[2][4];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
            ldmatrix_x4(qbase + sw128(rt * 16 + (lane & 15), hb * 4 + ks * 2 + (lane >> 4)), qf[ks][0], qf[ks][1],
                        qf[ks][2], qf[ks][3]);
        const int tq0 = y0 * a.W + rt * 16 + g, tq1 = tq0 + 8;  // query tokens of rows g, g+8
        const float *lwp = lw + (a.per_head ? hb * a.R * a.R : 0);
        const float *lw0 = lwp + (tq0 < a.N ? reg[tq0] : 0) * a.R;
        const float *lw1 = lwp + (tq1 < a.N ? reg[tq1] : 0) * a.R;
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
        float o[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

        for (int kb = 0; kb < a.npad; kb += 64) {
            const int nk = min(64, a.npad - kb);  // multiple of 16
            float sc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = -INFINITY;
                if (nt * 8 < nk) {
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(kbase + sw128(kb + nt * 8 + (lane & 7), hb * 4 + (lane >> 3)), b0, b1, b2, b3);
                    mma_bf16_16816(acc, qf[0], b0, b1);
                    mma_bf16_16816(acc, qf[1], b2, b3);
                    const int key = kb + nt * 8 + 2 * t;
                    const int rk0 = reg[key], rk1 = reg[key + 1];
                    const bool in0 = key < a.N, in1 = key + 1 < a.N;
                    sc[nt][0] = in0 ? fmaf(acc[0], a.scale_log2, lw0[rk0]) : -INFINITY;
                    sc[nt][1] = in1 ? fmaf(acc[1], a.scale_log2, lw0[rk1]) : -INFINITY;
                    sc[nt][2] = in0 ? fmaf(acc[2], a.scale_log2, lw1[rk0]) : -INFINITY;
                    sc[nt][3] = in1 ? fmaf(acc[3], a.scale_log2, lw1[rk1]) : -INFINITY;
                }
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
            }
            const float mn0 = fmaxf(m[0], quad_max(mx0)), mn1 = fmaxf(m[1], quad_max(mx1));
            // a row with no unmasked key so far keeps m = -inf: nothing to rescale, p = 0
            const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
            rescale(o, l, mn0 == -INFINITY ? 1.f : fast_exp2(m[0] - mn0), mn1 == -INFINITY ? 1.f : fast_exp2(m[1] - mn1));
            m[0] = mn0;
            m[1] = mn1;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                sc[nt][0] = fast_exp2(sc[nt][0] - base0);
                sc[nt][1] = fast_exp2(sc[nt][1] - base0);
                sc[nt][2] = fast_exp2(sc[nt][2] - base1);
                sc[nt][3] = fast_exp2(sc[nt][3] - base1);
                l[0] += sc[nt][0] + sc[nt][1];
                l[1] += sc[nt][2] + sc[nt][3];
            }
            if (nk == 64)
                pv_product<4>(o, sc, vbase, kb, hb, lane);
            else if (nk == 48)
                pv_product<3>(o, sc, vbase, kb, hb, lane);
            else if (nk == 32)
                pv_product<2>(o, sc, vbase, kb, hb, lane);
            else
                pv_product<1>(o, sc, vbase, kb, hb, lane);
        }
        __syncwarp();
        stage_output(qbase, o, l, rt * 16, hb, lane);  // overwrites only this warp's rows/head of the query tile
    }
    fence_async_shared();
    __syncthreads();
    if (threadIdx.x == 0 && alive && y0 < a.Hm) {  // a band wholly below a padded image stores nothing
        for (int j = 0; j < cpb; ++j) tma_store_4d(&tout, sQ + j * qtile, (cb0 + j) * 64, 0, y0, b);
        tma_store_commit();
        tma_store_wait_read();
    }
}

bool dense_mma_supports(const Geometry &g)
{
    return g.hd == 32 && g.C % 64 == 0 && g.R <= 64 && g.N <= 256 && g.W <= 256 && g.H <= 256;
}

int dense_mma_rows_per_split(const Geometry &g, int num_sms)
{
    const long long base = (long long)g.B * (g.C / 64);
    int nsplit = (int)((2LL * num_sms + base - 1) / base);
    if (nsplit < 1) nsplit = 1;
    if (nsplit > g.H) nsplit = g.H;
    return (g.H + nsplit - 1) / nsplit;
}

static size_t dense_smem_bytes(const Geometry &g, int rows_per_split, int cpb = 1, bool route = false,
                               bool per_head = false)
{
    const int nq = rows_per_split * g.W, nqpad = (nq + 15) & ~15;
    const int npad = (g.N + 15) & ~15;
    const int nct = g.C / 64 / cpb;
    const size_t routing = route ? (size_t)cpb * 64 * kDensePartPad * 4 + (size_t)((g.R + nct - 1) / nct) * 64 * 8 : 0;
    return 1024 + (size_t)cpb * (nqpad + 2 * npad) * kRowBytes + routing + (size_t)(per_head ? 2 : 1) * g.R * g.R * 4 +
           npad + 16;
}

static void fill_dense_args(DenseArgs &a, const int32_t *idx, const Geometry &g, int rows_per_split, unsigned *err,
                            bool inputs_ready, int Hm)
{
    a.inputs_ready = inputs_ready ? 1 : 0;
    a.Hm = Hm;
    a.idx = idx;
    a.idx_out = nullptr;
    a.err = err;
    a.H = g.H;
    a.W = g.W;
    a.n_win = g.n_win;
    a.topk = g.topk;
    a.R = g.R;
    a.hr = g.hr;
    a.wr = g.wr;
    a.N = g.N;
    a.npad = (g.N + 15) & ~15;
    a.ncb = g.C / 64;
    a.cpb = 1;
    a.rows_per_split = rows_per_split;
    a.nsplit = (g.H + rows_per_split - 1) / rows_per_split;
    a.per_head = 0;
    a.heads = g.heads;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    a.route_scale = (float)(1.0 / sqrt((double)g.C));
}

cudaError_t launch_attend_dense_mma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                    const CUtensorMap &tout, const int32_t *idx, const Geometry &g, int rows_per_split,
                                    unsigned *err, bool inputs_ready, int Hm, cudaStream_t stream, bool per_head)
{
    DenseArgs a;
    fill_dense_args(a, idx, g, rows_per_split, err, inputs_ready, Hm);
    a.per_head = per_head ? 1 : 0;
    const size_t smem = dense_smem_bytes(g, rows_per_split, 1, false, per_head);
    const long long blocks = (long long)g.B * a.ncb * a.nsplit;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // three CTAs per SM when their shared memory fits (227 KB per SM, 1 KB reserved per CTA)
    if (3 * (smem + 1024) <= 227 * 1024) {
        static int granted3[64] = {0};
        cudaError_t e = ensure_smem_limit(attend_dense_mma_kernel<3, false>, smem, granted3);
        if (e != cudaSuccess) return e;
        return launch_pdl(attend_dense_mma_kernel<3, false>, dim3((unsigned)blocks), dim3(256), smem, stream, tq, tk,
                          tv, tout, a);
    }
    static int granted[64] = {0};
    cudaError_t e = ensure_smem_limit(attend_dense_mma_kernel<2, false>, smem, granted);
    if (e != cudaSuccess) return e;
    return launch_pdl(attend_dense_mma_kernel<2, false>, dim3((unsigned)blocks), dim3(256), smem, stream, tq, tk, tv,
                      tout, a);
}

// 64-channel blocks per CTA of the fused kernel: two when the channel blocks pair up and two
// CTAs of that size fit on an SM, so that half as many CTAs (and clusters half as wide) carry
// the image; else one.
static int route_dense_cpb(const Geometry &g)
{
    const int ncb = g.C / 64;
    if (ncb % 2 == 0 && ncb / 2 <= kRouteDenseMaxCluster && 2 * (dense_smem_bytes(g, g.H, 2, true) + 1024) <= 227 * 1024)
        return 2;
    return 1;
}

bool route_dense_supports(const Geometry &g, bool bf16)
{
    if (!bf16 || !dense_mma_supports(g) || g.rs != 1 || g.R > 64 || !route_tokens_mma_supports(g, bf16)) return false;
    const int cpb = route_dense_cpb(g);
    return g.C / 64 <= kDenseMaxBlocks && g.C / 64 / cpb <= kRouteDenseMaxCluster &&
           dense_smem_bytes(g, g.H, cpb, true) <= 227 * 1024;
}

cudaError_t launch_route_attend_dense(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                      const CUtensorMap &tout, int32_t *idx, const Geometry &g, unsigned *err,
                                      cudaStream_t stream)
{
    if (!route_dense_supports(g, true)) return cudaErrorInvalidConfiguration;
    DenseArgs a;
    fill_dense_args(a, nullptr, g, g.H, err, false, g.H);
    a.idx_out = idx;
    a.cpb = route_dense_cpb(g);
    const int nct = a.ncb / a.cpb;
    const size_t smem = dense_smem_bytes(g, g.H, a.cpb, true);
    const long long blocks = (long long)g.B * nct;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    static int granted[64] = {0};
    cudaError_t e = ensure_smem_limit(attend_dense_mma_kernel<2, true>, smem, granted);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)nct;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attend_dense_mma_kernel<2, true>, tq, tk, tv, tout, a);
}

}  // namespace bra
