// bra_routing.cuh -- device routines of the routing step: the 64-bit routing keys, the warp
// top-k selection, the affinity rows (several rows x several keys per lane) and the staging of
// mean rows into padded shared-memory rows. The CUDA-core routing kernels are built from these
// and sum in one order, so they give the same bits. The tensor-core routing kernels (bf16 MMAs
// for one-token regions, 3xTF32 for fp32 inputs) use the keys and the selection from here with
// their sums in another order; each serves every call of its shapes, through either routing
// entry point, so the index of a shape never depends on the entry point.
#pragma once

#include "bra_device.cuh"

namespace bra {

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

__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long x)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, off);
        x = y > x ? y : x;
    }
    return x;
}

// Selects the topk largest of a warp's keys (lane l holds the keys of positions e * 32 + l,
// e < E) and writes their regions to out[0 .. topk): rounds of warp argmax (ROUNDS) or a
// shuffle bitonic network over position p = e * 32 + lane.
template <int E, bool ROUNDS>
__device__ __forceinline__ void select_topk(unsigned long long (&key)[E], int topk, int32_t *out, int lane)
{
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

// Rows per warp pass of affinity_accumulate: NR rows x E keys x 4 partial sums stay in registers.
template <int E>
struct RowsPerPass {
    static constexpr int value = E <= 2 ? 2 : 1;
};

// Routing rows i < nr (nr <= NR) of one image, by one warp, over channels [0, cn) of the rows
// given: query mean row i at qrows + i * qstride, key mean row s at kbase + s * kstride. Lane l
// accumulates the affinities of regions s = e * 32 + l, e < E (R <= 32 E), for all NR rows at
// once: every pair (row, s) is a dot product of four interleaved partial sums over the channels
// in order (channel c into sum c % 4), so that calls over consecutive channel windows continue
// the same sum;
// the NR x E products only run side by side, so that each 16-byte key load serves NR rows and
// the loads of consecutive channel steps overlap.
template <int E, int NR>
__device__ __forceinline__ void affinity_accumulate(float (&acc)[NR][E][4], const float *qrows, int qstride, int nr,
                                                    const float *kbase, int kstride, int R, int cn, int lane)
{
    int krow[E], qrow[NR];  // element offsets of the rows
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int s = e * 32 + lane;
        krow[e] = (s < R ? s : 0) * kstride;  // lanes past R compute a discarded key
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) qrow[i] = (i < nr ? i : 0) * qstride;
    constexpr int kUnroll = E >= 8 ? 2 : 4;  // keeps the E x kUnroll key loads in registers
#pragma unroll kUnroll
    for (int c = 0; c < cn; c += 4) {
        float4 y[E];
#pragma unroll
        for (int e = 0; e < E; ++e) y[e] = *reinterpret_cast<const float4 *>(kbase + krow[e] + c);
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            const float4 x = *reinterpret_cast<const float4 *>(qrows + qrow[i] + c);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                acc[i][e][0] = fmaf(x.x, y[e].x, acc[i][e][0]);
                acc[i][e][1] = fmaf(x.y, y[e].y, acc[i][e][1]);
                acc[i][e][2] = fmaf(x.z, y[e].z, acc[i][e][2]);
                acc[i][e][3] = fmaf(x.w, y[e].w, acc[i][e][3]);
            }
        }
    }
}

// The affinities of rows i < nr from their partial sums, combined as (s0 + s1) + (s2 + s3), times
// C^-1/2, and their top-k, written to out + i * topk. The CUDA-core routing kernels go through
// affinity_accumulate and this function, so their index is the same bits whichever of them
// computed it.
template <int E, int NR, bool ROUNDS>
__device__ __forceinline__ void affinity_select(const float (&acc)[NR][E][4], int nr, int R, int topk, float scale,
                                                int32_t *out, int lane)
{
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        if (i >= nr) break;
        unsigned long long key[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int s = e * 32 + lane;
            const float d = (acc[i][e][0] + acc[i][e][1]) + (acc[i][e][2] + acc[i][e][3]);
            key[e] = s < R ? routing_key(d * scale, s) : 0ull;
        }
        select_topk<E, ROUNDS>(key, topk, out + (size_t)i * topk, lane);
    }
}

// 16 bytes of S elements as fp32 (bf16 widens exactly).
__device__ __forceinline__ void store_as_f32(float *d, uint4 v, float)
{
    *reinterpret_cast<float4 *>(d) = make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                                                 __uint_as_float(v.w));
}
__device__ __forceinline__ void store_as_f32(float *d, uint4 v, __nv_bfloat16)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
    *reinterpret_cast<float4 *>(d) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4 *>(d + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// Copies channels [c0, c0 + cn) (multiples of 16 bytes of S) of rows0 rows from src0 and then of
// rows1 rows from src1 (row stride C elements) as fp32 to consecutive rows of dst (row stride
// dst_stride), all threads of the CTA, eight 16-byte loads in flight per thread. With L2 set,
// the loads bypass L1 (ld.global.cg): the rows were written by other CTAs of this grid.
template <bool L2, typename S>
__device__ __forceinline__ void stage_rows(const S *__restrict__ src0, int rows0, const S *__restrict__ src1, int rows1,
                                           float *dst, int C, int c0, int cn, int dst_stride)
{
    constexpr int V = 16 / sizeof(S);
    const int cv = cn / V;  // 16-byte vectors per row window
    const int nrows = rows0 + rows1;
    auto load = [&](int row, int col) -> uint4 {
        const S *src = row < rows0 ? src0 + (size_t)row * C : src1 + (size_t)(row - rows0) * C;
        const uint4 *p = reinterpret_cast<const uint4 *>(src + c0 + col * V);
        return L2 ? __ldcg(p) : __ldg(p);
    };
    if (blockDim.x % cv == 0) {
        // each thread keeps one column and steps through the rows: no division per element
        const int col = threadIdx.x % cv, step = blockDim.x / cv;
        for (int r0 = threadIdx.x / cv; r0 < nrows; r0 += 8 * step) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (r0 + u * step < nrows) v[u] = load(r0 + u * step, col);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (r0 + u * step < nrows) store_as_f32(dst + (size_t)(r0 + u * step) * dst_stride + col * V, v[u], S());
        }
        return;
    }
    const int total = nrows * cv;
    for (int e0 = threadIdx.x; e0 < total; e0 += 8 * blockDim.x) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * blockDim.x;
            if (e < total) v[u] = load(e / cv, e % cv);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * blockDim.x;
            if (e < total) store_as_f32(dst + (size_t)(e / cv) * dst_stride + (e % cv) * V, v[u], S());
        }
    }
}

}  // namespace bra
