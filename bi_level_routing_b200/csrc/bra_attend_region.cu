// bra_attend_region.cu -- gather attention for regions of 4 tokens (bf16, head_dim 32), with
// the heads stacked into the rows of the tensor-core tiles.
//
// What it computes ("从零构建BiFormer", §2.2 TokenAttention; "医学图像分割模块：BiFormer /
// 双层路由注意力", §五 steps ⑤-⑦): for every query token of region r and every head, softmax
// (scale head_dim^-1/2) over the tokens of the regions idx[b, r, 0..topk-1] (a region listed
// twice counts twice; an index outside [0, R) is skipped and flagged), then the weighted sum of
// their values, accumulated in fp32, out rounded to bf16.
//
// Why stacked heads: an mma.sync tile has 16 rows, but a region has only 4 query tokens, and
// tokens of different regions attend to different keys. The 4 tokens x 4 heads of one region
// do share their keys, so they make one 16-row tile: row i is token i % 4 of head i / 4. For
// Q K^T the tile's A operand is block-diagonal over the 128 channels of the 4 heads (a row
// holds its own head's 32 channels and zeros elsewhere), so each row meets only its head's
// channels of K; for P V each row keeps only its head's 32 output channels. The MMAs do 4x the
// useful work, which the tensor pipe has to spare; every score and every exponential computed
// is used, where masked dense attention over the whole image discards most of them.
//
// One CTA per (image, group of 4 heads = 128 channels, split of the query regions): one TMA
// load per tensor stages the image's q, k and v for those channels in shared memory (5-D box:
// two 64-channel tiles of H x W rows, 128-byte swizzle); warp w of 12 then takes query regions
// w, w + 12, ... (of its split). Per region it gathers the routed keys straight from shared
// memory: ldmatrix reads rows at per-lane addresses, so key j of the tile is token j % 4 of
// region idx[b, r, j / 4] wherever it sits. Keys go in chunks of 64 with an online softmax.
// Every wait is bounded (kErrTimeout).
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

namespace {

constexpr int kRegionWarps = 12;

struct RegionArgs {
    const int32_t *idx;
    unsigned *err;
    __nv_bfloat16 *out;
    int H, W, C, n_win, topk, R, hr, wr, N;
    int wshift;   // log2(wr)
    int ngroups;  // C / 128
    int nsplit;   // CTAs per (image, group); query regions are dealt among them
    int keys;     // 4 topk rounded up to a multiple of 16
    int Hm, Wm;   // the image in memory (H, W: the region grid, which may cover more)
    float scale_log2;
    int inputs_ready;  // q, k, v may be loaded before the wait for the previous kernel
};

// bytes of one staged tensor (two 64-channel tiles of N rows, then one spare row: zeros, in the
// V buffer), rounded up to the 1024-byte period of the swizzle
__host__ __device__ inline size_t region_tile_bytes(int N) { return ((size_t)(2 * N + 1) * 128 + 1023) & ~(size_t)1023; }

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float quad_max_f(float x)
{
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ float quad_sum_f(float x)
{
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

}  // namespace

__global__ void __launch_bounds__(32 * kRegionWarps, 1) attend_region_mma_kernel(
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const RegionArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const size_t tile = region_tile_bytes(a.N);
    uint8_t *sQ = smem, *sK = smem + tile, *sV = smem + 2 * tile;
    int *row0 = reinterpret_cast<int *>(smem + 3 * tile);  // [R] row of each region's first token
    int *sidx = row0 + a.R;                                  // [R * topk] this image's routing index
    uint64_t *bar = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(sidx + a.R * a.topk) + 7) & ~uintptr_t(7));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int item = blockIdx.x;
    const int split = item % a.nsplit;
    item /= a.nsplit;
    const int grp = item % a.ngroups;
    const int b = item / a.ngroups;

    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    // q, k and v: before the wait for the previous kernel when that kernel is the routing step of
    // the same forward pass (it already waited for their producers), else after it
    if (!a.inputs_ready) grid_dependency_wait();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(3 * 2 * a.N * 128));
        tma_load_5d(sQ, &tq, 0, 0, 0, 2 * grp, b, bar);
        tma_load_5d(sK, &tk, 0, 0, 0, 2 * grp, b, bar);
        tma_load_5d(sV, &tv, 0, 0, 0, 2 * grp, b, bar);
    }
    if (a.inputs_ready) grid_dependency_wait();  // idx comes from the previous kernel
    // V row 2 N: zeros, read for padding keys and skipped regions (their p is 0, and 0 times a
    // non-finite value in a real row would not be)
    if (threadIdx.x < 8) reinterpret_cast<uint4 *>(sV + (size_t)2 * a.N * 128)[threadIdx.x] = make_uint4(0, 0, 0, 0);
    for (int s = threadIdx.x; s < a.R; s += blockDim.x) {
        const int ry = s / a.n_win;
        row0[s] = ry * a.hr * a.W + (s - ry * a.n_win) * a.wr;
    }
    const int32_t *gidx = a.idx + (int64_t)b * a.R * a.topk;
    for (int e = threadIdx.x; e < a.R * a.topk; e += blockDim.x) {
        const int s = gidx[e];
        const bool ok = s >= 0 && s < a.R;
        if (!ok && grp == 0 && split == 0) flag_error(a.err, kErrIndex);
        sidx[e] = ok ? s : -1;
    }
    __syncthreads();
    const bool alive = mbar_wait(bar, 0, a.err);

    const int g = lane >> 2, t4 = lane & 3;
    const int hA = g >> 2, hB = 2 + (g >> 2);  // heads of this lane's rows g and g + 8
    const uint32_t qbase = smem_u32(sQ), kbase = smem_u32(sK), vbase = smem_u32(sV);
    const int n_keys = 4 * a.topk;
    // row offset of token t of a region from its first token (wr = 1 << wshift is 1, 2 or 4)
    auto toff = [&](int t) -> int { return (t >> a.wshift) * a.W + (t & (a.wr - 1)); };
    // address of channel c (0..127, even) of staged row n: channel block c / 64, 16-byte chunk
    auto addr = [&](uint32_t base, int n, int c) -> uint32_t {
        return base + sw128((c >> 6) * a.N + n, (c & 63) >> 3) + (c & 7) * 2;
    };

    for (int r = split + a.nsplit * warp; alive && r < a.R; r += a.nsplit * kRegionWarps) {
        // Q of this lane's rows: token g % 4 of region r, heads hA (row g) and hB (row g + 8);
        // per head two 16-channel k steps, each a low and a high pair of channels
        const int qrow = row0[r] + toff(g & 3);
        uint32_t qa[2][2], qb[2][2];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            qa[ks][0] = ld_shared_u32(addr(qbase, qrow, 32 * hA + 16 * ks + 2 * t4));
            qa[ks][1] = ld_shared_u32(addr(qbase, qrow, 32 * hA + 16 * ks + 2 * t4 + 8));
            qb[ks][0] = ld_shared_u32(addr(qbase, qrow, 32 * hB + 16 * ks + 2 * t4));
            qb[ks][1] = ld_shared_u32(addr(qbase, qrow, 32 * hB + 16 * ks + 2 * t4 + 8));
        }
        const int *ridx = sidx + r * a.topk;
        // bit j: routed region j of this row is in range (topk <= 64)
        const uint32_t ok_lo = __ballot_sync(0xffffffffu, lane < a.topk && ridx[lane] >= 0);
        const uint32_t ok_hi = __ballot_sync(0xffffffffu, lane + 32 < a.topk && ridx[lane + 32] >= 0);
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
        float oA[4][2], oB[4][2];  // row g: head hA's 32 channels; row g + 8: head hB's
#pragma unroll
        for (int i = 0; i < 4; ++i) oA[i][0] = oA[i][1] = oB[i][0] = oB[i][1] = 0.f;

        for (int kc = 0; kc < a.keys; kc += 64) {
            const int nk = min(64, a.keys - kc);  // a multiple of 16
            // staged row of keys kc + lane and kc + 32 + lane (-1: padding or a skipped region);
            // the ldmatrix rows of K and V come from these by shuffles
            int kra, krb;
            {
                const int k0 = kc + lane, k1 = kc + 32 + lane;
                const int s0 = k0 < n_keys ? ridx[k0 >> 2] : -1, s1 = k1 < n_keys ? ridx[k1 >> 2] : -1;
                kra = s0 >= 0 ? row0[s0] + toff(k0 & 3) : -1;
                krb = s1 >= 0 ? row0[s1] + toff(k1 & 3) : -1;
            }
            float sc[8][4];
            int krow[8];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                // this lane's ldmatrix row: key kc + 8 nt + (lane & 7); masked keys read row 0
                const int kr = __shfl_sync(0xffffffffu, nt < 4 ? kra : krb, (8 * nt + (lane & 7)) & 31);
                krow[nt] = kr >= 0 ? kr : 0;
            }
            // S = Q K^T for the chunk's 8-key tiles: per head, four tiles' ldmatrix first, then
            // their MMAs side by side (independent accumulators)
#pragma unroll
            for (int hk = 0; hk < 4; ++hk) {
#pragma unroll
                for (int n0 = 0; n0 < 8; n0 += 4) {  // four tiles at a time
                    uint32_t bk[4][4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if ((n0 + i) * 8 < nk)
                            ldmatrix_x4(kbase + sw128((hk >> 1) * a.N + krow[n0 + i], 4 * (hk & 1) + (lane >> 3)),
                                        bk[i][0], bk[i][1], bk[i][2], bk[i][3]);
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        // block-diagonal A: row g holds head hA's channels, row g + 8 head hB's
                        const uint32_t af[4] = {hk == hA ? qa[ks][0] : 0u, hk == hB ? qb[ks][0] : 0u,
                                                hk == hA ? qa[ks][1] : 0u, hk == hB ? qb[ks][1] : 0u};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if ((n0 + i) * 8 < nk) mma_bf16_16816(sc[n0 + i], af, bk[i][2 * ks], bk[i][2 * ks + 1]);
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                // keys kc + 8 nt + 2 t4 and + 1 lie in one region: both valid or both not
                const int kk = kc + nt * 8 + 2 * t4, j = kk >> 2;
                const bool ok = nt * 8 < nk && kk < n_keys && (((j < 32 ? ok_lo >> j : ok_hi >> (j - 32)) & 1u) != 0);
#pragma unroll
                for (int j = 0; j < 4; ++j) sc[nt][j] = ok ? sc[nt][j] * a.scale_log2 : -INFINITY;
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
            }
            const float mn0 = fmaxf(m[0], quad_max_f(mx0)), mn1 = fmaxf(m[1], quad_max_f(mx1));
            // a row with no valid key so far keeps m = -inf: nothing to rescale, p = 0
            const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
            const float c0 = mn0 == -INFINITY ? 1.f : fast_exp2(m[0] - mn0);
            const float c1 = mn1 == -INFINITY ? 1.f : fast_exp2(m[1] - mn1);
            m[0] = mn0;
            m[1] = mn1;
            l[0] *= c0;
            l[1] *= c1;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                oA[i][0] *= c0;
                oA[i][1] *= c0;
                oB[i][0] *= c1;
                oB[i][1] *= c1;
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                sc[nt][0] = fast_exp2(sc[nt][0] - base0);
                sc[nt][1] = fast_exp2(sc[nt][1] - base0);
                sc[nt][2] = fast_exp2(sc[nt][2] - base1);
                sc[nt][3] = fast_exp2(sc[nt][3] - base1);
                l[0] += sc[nt][0] + sc[nt][1];
                l[1] += sc[nt][2] + sc[nt][3];
            }
            // O += P V over this chunk's keys: P from the score registers (bf16), V rows
            // gathered by ldmatrix (key kc + 16 kk + (lane & 15) for this lane's row address)
            uint32_t pa[4][4];
            int vrow[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                pa[kk][0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
                pa[kk][1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
                pa[kk][2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                pa[kk][3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
                vrow[kk] = __shfl_sync(0xffffffffu, kk < 2 ? kra : krb, (16 * kk + (lane & 15)) & 31);
            }
            // two 16-channel pairs at a time: four independent accumulators per key step
#pragma unroll
            for (int np0 = 0; np0 < 8; np0 += 2) {  // output channels 16 np0 .. 16 np0 + 31
                float acc[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (16 * kk < nk) {
#pragma unroll
                        for (int d = 0; d < 2; ++d) {
                            const int np = np0 + d;
                            const int vr = vrow[kk] >= 0 ? (np >> 2) * a.N + vrow[kk] : 2 * a.N;
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4_trans(vbase + sw128(vr, 2 * (np & 3) + (lane >> 4)), b0, b1, b2, b3);
                            mma_bf16_16816(acc[2 * d], pa[kk], b0, b1);
                            mma_bf16_16816(acc[2 * d + 1], pa[kk], b2, b3);
                        }
                    }
                }
                // n tiles 2 np and 2 np + 1 belong to head np / 2: rows of head hA (np < 4) take
                // their row g values, rows of head hB (np >= 4) their row g + 8 values
#pragma unroll
                for (int d = 0; d < 2; ++d) {
                    const int np = np0 + d, h = np >> 1, i0 = (2 * np) & 3;
                    if (h == hA) {
                        oA[i0][0] += acc[2 * d][0];
                        oA[i0][1] += acc[2 * d][1];
                        oA[i0 + 1][0] += acc[2 * d + 1][0];
                        oA[i0 + 1][1] += acc[2 * d + 1][1];
                    }
                    if (h == hB) {
                        oB[i0][0] += acc[2 * d][2];
                        oB[i0][1] += acc[2 * d][3];
                        oB[i0 + 1][0] += acc[2 * d + 1][2];
                        oB[i0 + 1][1] += acc[2 * d + 1][3];
                    }
                }
            }
        }
        // normalise and store: row g -> token qrow, channels 128 grp + 32 hA + 8 i + 2 t4
        const float l0 = quad_sum_f(l[0]), l1 = quad_sum_f(l[1]);
        const float inv0 = l0 > 0.f ? __fdividef(1.f, l0) : 0.f, inv1 = l1 > 0.f ? __fdividef(1.f, l1) : 0.f;
        const int qy = qrow / a.W, qx = qrow - qy * a.W;  // qrow: a row of the staged (grid-sized) map
        if (qy < a.Hm && qx < a.Wm) {  // tokens of a padded map outside the image are not stored
            __nv_bfloat16 *dst = a.out + (((int64_t)b * a.Hm + qy) * a.Wm + qx) * a.C + 128 * grp + 2 * t4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                *reinterpret_cast<uint32_t *>(dst + 32 * hA + 8 * i) = pack_bf16x2(oA[i][0] * inv0, oA[i][1] * inv0);
                *reinterpret_cast<uint32_t *>(dst + 32 * hB + 8 * i) = pack_bf16x2(oB[i][0] * inv1, oB[i][1] * inv1);
            }
        }
    }
}

bool region_mma_supports(const Geometry &g)
{
    return g.hd == 32 && g.C % 128 == 0 && g.rs == 4 && g.N <= 256 && g.W <= 256 && g.H <= 256 && g.topk <= 64;
}

cudaError_t launch_attend_region_mma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                     const int32_t *idx, void *out, const Geometry &g, int H, int W, int num_sms,
                                     unsigned *err, bool inputs_ready, cudaStream_t stream)
{
    RegionArgs a;
    a.inputs_ready = inputs_ready ? 1 : 0;
    a.Hm = H;
    a.Wm = W;
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
    a.N = g.N;
    a.wshift = g.wr == 4 ? 2 : (g.wr == 2 ? 1 : 0);  // rs = 4: wr is 1, 2 or 4
    a.ngroups = g.C / 128;
    a.keys = (4 * g.topk + 15) & ~15;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.hd));
    // one CTA per SM (shared memory); split the query regions when the images and head groups
    // alone leave SMs idle
    const long long base = (long long)g.B * a.ngroups;
    int nsplit = (int)(num_sms / (base > 0 ? base : 1));
    if (nsplit < 1) nsplit = 1;
    if (nsplit > g.R) nsplit = g.R;
    a.nsplit = nsplit;
    const long long blocks = base * nsplit;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const size_t smem = 1024 + 3 * region_tile_bytes(g.N) + 4 * (size_t)g.R * (1 + g.topk) + 16;
    static int granted[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)smem > granted[dev]) {
        e = cudaFuncSetAttribute(attend_region_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        granted[dev] = (int)smem;
    }
    return launch_pdl(attend_region_mma_kernel, dim3((unsigned)blocks), dim3(32 * kRegionWarps), smem, stream, tq, tk,
                      tv, a);
}

}  // namespace bra
