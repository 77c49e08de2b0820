// bra_launch.h -- host-side launchers of the BRA kernels (internal to libbra.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "bra.h"

namespace bra {

// Bits of the sticky device error word.
constexpr unsigned kErrIndex = 1u;    // an idx entry outside [0, R) was skipped
constexpr unsigned kErrTimeout = 2u;  // a bounded wait gave up

// Derived sizes of one call: R = n_win^2 regions of rs = hr * wr tokens, hd = C / heads.
struct Geometry {
    int B, H, W, C, heads, n_win, topk;
    int R, hr, wr, rs, hd, N;
};

// Launches `kernel` on `stream` with programmatic stream serialization: the grid may be
// scheduled as soon as the previous kernel's blocks have exited, and waits in
// grid_dependency_wait() for that kernel's completion before its dependent reads, so the launch
// latency and the prologue overlap the previous kernel's drain.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Sets the message bra_last_error_message returns on this thread.
void set_last_error(const std::string &msg);

// Grid of a persistent attention kernel over `nitems` work items: `per_sm` CTAs per SM, at most
// one CTA per item, and at most the cap set by bra_set_max_ctas (0 = none).
int persistent_grid(long long nitems, int num_sms, int per_sm = 2);

// The argument checks of bra_route (shape, NULL pointers, alignment); fills g.
bra_status check_route_args(const void *q, const void *k, const int32_t *idx, int B, int H, int W, int C, int n_win,
                            int topk, bra_dtype dtype, Geometry *g);

// Region means of q and k (fp32, [B, R, C] each) into qm and km. One region row segment
// (wr tokens x C channels) may hold at most kMaxMeansVectors 16-byte vectors.
constexpr int kMaxMeansVectors = 2048;
cudaError_t launch_region_means(const void *q, const void *k, float *qm, float *km, const Geometry &g,
                                bool bf16, int num_sms, cudaStream_t stream);


// topk rounds of argmax cost about topk * (E + 20) instructions; the bitonic network
// log2(P) (log2(P) + 1) / 2 stages of about 8 E.
inline bool topk_by_rounds(int E, int topk)
{
    int lg = 5;
    while ((1 << lg) < 32 * E) ++lg;
    const long long stages = (long long)lg * (lg + 1) / 2;
    return (long long)topk * (E + 20) <= stages * E * 8;
}

// Affinity rows and top-k straight from q and k when a region is one token (rs == 1, R <= 256):
// the means are the tokens, widened exactly to fp32, so the index is the same as from the means.
cudaError_t launch_route_topk_tokens(const void *q, const void *k, int32_t *idx, const Geometry &g, bool bf16,
                                     cudaStream_t stream);
// The shapes the bf16 tensor-core kernel of that step serves (rs == 1, R <= 64, C % 32 == 0).
bool route_tokens_mma_supports(const Geometry &g, bool bf16);

// Affinity rows and top-k: idx[b, r, :] from qm, km.
cudaError_t launch_route_topk(const float *qm, const float *km, int32_t *idx, const Geometry &g,
                              cudaStream_t stream);

// Per-head routing ("医学图像分割模块", §五 steps ③④): idx [B, heads, R, topk] from the fp32
// region means (route_heads) or, for one-token regions, from q and k themselves (..._tokens).
// Needs R <= 256 and head slices on 16-byte boundaries (route_heads_supports).
bool route_heads_supports(const Geometry &g, bool bf16);
cudaError_t launch_route_heads(const float *qm, const float *km, int32_t *idx, const Geometry &g, cudaStream_t stream);
cudaError_t launch_route_heads_tokens(const void *q, const void *k, int32_t *idx, const Geometry &g, bool bf16,
                                      cudaStream_t stream);

// Region means of a map padded to the region grid g (g.H = n_win hr >= H, g.W = n_win wr >= W):
// tokens outside the H x W image count as zeros (auto_pad).
cudaError_t launch_region_means_padded(const void *q, const void *k, float *qm, float *km, const Geometry &g, int H,
                                       int W, bool bf16, cudaStream_t stream);

// Attention on CUDA cores with the routed key and value rows staged in shared memory: any dtype,
// head size up to kSimtMaxHeadDim, idx shared ([B, R, topk]) or per head ([B, heads, R, topk]),
// and maps padded to the region grid g (tokens at y >= H or x >= W are zeros; H = g.H, W = g.W
// for an unpadded call; q, k, v, out are [B, H, W, C]).
cudaError_t launch_attend_staged(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                                 const Geometry &g, int H, int W, bool per_head, bool bf16, unsigned *err,
                                 cudaStream_t stream);

// LePE epilogue: y = x + 5x5 depthwise conv(x) (zero padding 2) + bias; x, y [B, H, W, C] of the
// element type, weight fp32 [C, 5, 5], bias fp32 [C]; C a multiple of 16 bytes of elements.
bool lepe_supports(int C, bool bf16);
cudaError_t launch_lepe(const void *x, const float *weight, const float *bias, void *y, int B, int H, int W, int C,
                        bool bf16, cudaStream_t stream);

// Backward of the token attention with idx fixed: dq, dk, dv (fp32 [B, H, W, C]) of
// sum(dout * out); clears dk and dv (memset nodes), then one kernel. Needs hd % 8 == 0, rs <= 256.
bool attend_backward_supports(const Geometry &g);
cudaError_t launch_attend_backward(const void *q, const void *k, const void *v, const int32_t *idx, const void *dout,
                                   float *dq, float *dk, float *dv, const Geometry &g, bool bf16, unsigned *err,
                                   cudaStream_t stream);

// One thread waits on an mbarrier that never completes, with the library's bounded wait given
// limit_ns; it gives up and sets kErrTimeout in *err.
cudaError_t launch_wait_timeout(unsigned *err, unsigned long long limit_ns, cudaStream_t stream);

// Largest R the routing kernel handles.
constexpr int kMaxRegions = 1024;

// Generic attention on CUDA cores (fp32 or bf16, hd <= kSimtMaxHeadDim).
constexpr int kSimtMaxHeadDim = 128;
cudaError_t launch_attend_simt(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                               const Geometry &g, bool bf16, unsigned *err, cudaStream_t stream);

// Tensor-core attention kernels (bf16, hd == 32, C % 64 == 0). The tensor maps describe
// q, k, v, out as 4-D (C, W, H, B) bf16 tensors, 128-byte swizzle (except the gather kernel's
// q, k and v maps, 5-D, below); box sizes as each launcher's comment states. g is the region
// grid; H, W (arguments of the launchers that take them, and the maps' dimensions) the image in
// memory, smaller than the grid for a padded map (auto_pad): boxes that reach past the image read
// zeros, and rows outside it are not stored.
bool gather_mma_supports(const Geometry &g);
bool dense_mma_supports(const Geometry &g);

// Stacked-head gather attention for 4-token regions (bf16, hd == 32, C % 128 == 0, N <= 256,
// topk <= 64). Maps: q, k, v as 5-D views, box (64, W, H, 2, 1).
bool region_mma_supports(const Geometry &g);
// inputs_ready (here and for the dense kernel): q, k and v may be loaded before the kernel waits
// for its predecessor on the stream (true when that predecessor is the routing kernel of the same
// forward pass, which already waited for their producers); idx is read after the wait.
cudaError_t launch_attend_region_mma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                     const int32_t *idx, void *out, const Geometry &g, int H, int W, int num_sms,
                                     unsigned *err, bool inputs_ready, cudaStream_t stream);

// Box of the gather kernel's q, k and v maps: (64 channels, wr, hr, NCB channel blocks, 1 image)
// on the 5-D view (channel in block, x, y, channel block, image) of [B, H, W, C], so that one
// TMA load brings a region's NCB 64-channel tiles, one after the other. Its out map is 4-D,
// box (64, wr, hr, 1).
void gather_mma_box(const Geometry &g, int box[5]);
cudaError_t launch_attend_gather_mma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                     const CUtensorMap &tout, const int32_t *idx, void *out, const Geometry &g, int H,
                                     int W, int num_sms, unsigned *err, cudaStream_t stream,
                                     bool per_head = false);

// tcgen05 gather attention for 64-token regions (bf16, hd == 32, C % 64 == 0). Maps: q, k, v
// with box (64, wr, hr, 1).
bool gather_umma_supports(const Geometry &g);
cudaError_t launch_attend_gather_umma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                      const int32_t *idx, void *out, const Geometry &g, int H, int W, int num_sms,
                                      unsigned *err, cudaStream_t stream);

// Boxes of the dense kernel: q and out (64, W, rows_per_split, 1); k and v (64, W, H, 1).
// per_head: idx is [B, heads, R, topk] and each head of a 64-channel block is masked by its own
// routing counts.
int dense_mma_rows_per_split(const Geometry &g, int num_sms);
cudaError_t launch_attend_dense_mma(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                    const CUtensorMap &tout, const int32_t *idx, const Geometry &g,
                                    int rows_per_split, unsigned *err, bool inputs_ready, int Hm,
                                    cudaStream_t stream, bool per_head = false);

// The forward pass of one-token regions (bf16, R <= 64) in one kernel: the dense kernel with the
// routing step inside, launched as one thread-block cluster per image (at most
// kRouteDenseMaxCluster CTAs, one or two 64-channel blocks each). It writes idx [B, R, topk]
// with the same bits as the routing kernel of these shapes and out as the dense kernel does.
// Maps: q and out with box (64, W, H, 1), k and v likewise.
constexpr int kRouteDenseMaxCluster = 8;
bool route_dense_supports(const Geometry &g, bool bf16);
cudaError_t launch_route_attend_dense(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                      const CUtensorMap &tout, int32_t *idx, const Geometry &g, unsigned *err,
                                      cudaStream_t stream);

}  // namespace bra
