/*
 * bra.h -- C ABI of libbra.so: the forward pass of Bi-Level Routing Attention (BRA) on one
 * NVIDIA B200 (sm_100a).
 *
 * BRA, as defined by the BiFormer pages this library restates:
 *   1. cut the H x W feature map into n_win x n_win non-overlapping regions of
 *      rs = (H / n_win) * (W / n_win) tokens ("从零构建BiFormer", §1 region_partition;
 *      "手把手带你读懂BiFormer源码", §1.1 RegionPartition);
 *   2. region-mean descriptors qm, km of q and k ("手把手带你读懂BiFormer源码", §1.2 step 1);
 *   3. region affinity A = C^-1/2 qm km^T, R x R per image ("手把手带你读懂BiFormer源码",
 *      §1.2 step 2; "从静态到动态", §2.1 TopkRouting);
 *   4. routing index idx = the topk largest affinities of each row ("手把手带你读懂BiFormer源码",
 *      §1.2 step 3);
 *   5. for every query token of region r and every head: softmax attention, scale
 *      head_dim^-1/2, over the tokens of the regions idx[r][0..topk-1] only
 *      ("从零构建BiFormer", §2.2 TokenAttention; "医学图像分割模块：BiFormer / 双层路由注意力",
 *      §五 steps ⑤-⑦).
 * bra_route does steps 1-4, bra_attend step 5 and bra_forward all of them.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout. q, k, v and out are dense, contiguous [B, H, W, C] arrays (channels innermost,
 *   then x, then y, then image) in DEVICE memory, of element type `dtype`. Head j owns
 *   channels [j*hd, (j+1)*hd), hd = C / heads. Regions are numbered row-major over the
 *   n_win x n_win grid: region r = (y / (H/n_win)) * n_win + x / (W/n_win). idx is a dense
 *   int32 [B, R, topk] device array, R = n_win^2.
 * Routing order. Each idx row lists regions by affinity descending; equal affinities put
 *   the lower region index first; NaN affinities rank below every number. Routing is
 *   shared by all heads and uses the full-C region means, accumulated in fp32.
 * Precision. bf16 inputs are accumulated in fp32 (means, affinities, logits, softmax and
 *   the weighted sum); out is rounded to bf16 (nearest even). fp32 inputs: fp32 throughout.
 * Ownership. Every buffer belongs to the caller. Calls are asynchronous and ordered on
 *   `stream` (a cudaStream_t; NULL = the legacy default stream) on the current device;
 *   the library never synchronises, except bra_check_device_error and bra_forward_host.
 *   bra_route takes fp32 scratch for the region means, 2*B*R*C*4 bytes, from a
 *   stream-ordered pool the library keeps per device (cudaMallocAsync / cudaFreeAsync on
 *   `stream`); bra_forward keeps them in `out` instead, which the attention overwrites
 *   afterwards, and allocates nothing (when they fit: rs * sizeof(element) >= 8; one-token
 *   regions need no means).
 * Validation. Every argument is checked on the host before anything is launched; a
 *   rejected call launches nothing and returns BRA_ERR_INVALID_ARG: a NULL pointer (when
 *   B > 0), B < 0, H, W, C, heads, n_win or topk <= 0, H or W not a multiple of n_win,
 *   C not a multiple of heads, topk > R, a data pointer not 16-byte aligned, idx not
 *   4-byte aligned, C * sizeof(element) not a multiple of 16 bytes, an unknown dtype.
 *   B == 0 is an empty batch: nothing is launched and BRA_OK is returned.
 *   BRA_ERR_UNSUPPORTED: valid but outside this build's limits (R > 1024, hd > 128).
 *   BRA_ERR_CUDA: a CUDA call failed (the message is in bra_last_error_message()).
 * Device-side checks. bra_attend checks every idx entry on the device; an entry outside
 *   [0, R) is skipped (its region contributes no key; a query left with no key gets 0)
 *   and a sticky device error word is set, which bra_check_device_error reports as
 *   BRA_ERR_INDEX. A bounded wait that gave up sets BRA_ERR_TIMEOUT the same way.
 */
#ifndef BRA_H
#define BRA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BRA_OK = 0,
    BRA_ERR_INVALID_ARG = 1,
    BRA_ERR_UNSUPPORTED = 2,
    BRA_ERR_CUDA = 3,
    BRA_ERR_INDEX = 4,
    BRA_ERR_TIMEOUT = 5
} bra_status;

typedef enum { BRA_F32 = 0, BRA_BF16 = 1 } bra_dtype;

/* Which attention kernel bra_attend / bra_forward use. AUTO picks per shape; the others
   force one kernel (for tests and tuning) and make calls it cannot serve return
   BRA_ERR_UNSUPPORTED. */
typedef enum {
    BRA_ATTEND_AUTO = 0,
    BRA_ATTEND_SIMT = 1,      /* any dtype, hd <= 128: routed rows staged in shared memory, one
                                 thread per (query, head), CUDA cores */
    BRA_ATTEND_GATHER_MMA = 2,/* bf16, hd == 32, C % 64 == 0, rs % 16 == 0, rs <= 64: per-region
                                 tiles staged by TMA, tensor-core QK^T and PV */
    BRA_ATTEND_DENSE_MMA = 3, /* bf16, hd == 32, C % 64 == 0, R <= 64, H*W <= 256: the image's
                                 K/V staged once, masked by the routing multiplicities */
    BRA_ATTEND_GATHER_UMMA = 4,/* bf16, hd == 32, C % 64 == 0, rs == 64: per-region tiles staged
                                 by TMA, QK^T and PV on the tcgen05 tensor cores with TMEM
                                 accumulators, one softmax thread per query row */
    BRA_ATTEND_REGION_MMA = 5 /* bf16, hd == 32, C % 128 == 0, rs == 4, H*W <= 256, topk <= 64:
                                 the image's q, k, v for 4 heads staged once; tiles of 4 tokens
                                 x 4 heads of one region, routed keys gathered from shared
                                 memory */
} bra_attend_kernel;

/* Steps 1-4: idx[b, r, :] = routing index of region r of image b.
   q, k: device [B, H, W, C] of dtype. idx: device int32 [B, n_win^2, topk], written. */
bra_status bra_route(const void *q, const void *k, int32_t *idx, int B, int H, int W, int C, int n_win,
                     int topk, bra_dtype dtype, void *stream);

/* Step 5: out = token-to-token attention of every query over the routed regions' keys.
   q, k, v: device [B, H, W, C] of dtype. idx: device int32 [B, n_win^2, topk], read (any
   values: duplicates are gathered as often as they occur; out-of-range entries are
   skipped and flagged). out: device [B, H, W, C] of dtype, written; must not overlap the
   inputs. */
bra_status bra_attend(const void *q, const void *k, const void *v, const int32_t *idx, void *out, int B,
                      int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream);

/* Steps 1-5: bra_route then bra_attend on the same stream. idx is written (and then read).
   Where every region is one token (H = W = n_win), bf16, R <= 64 and the attention kernel in
   use is BRA_ATTEND_DENSE_MMA, both steps run in one kernel (one thread-block cluster per
   image); idx and out are then the same bits as from bra_route and bra_attend. */
bra_status bra_forward(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H,
                       int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream);

/* Steps 1-4 exactly like bra_route (same kernels, same idx), for callers that cannot
   allocate device memory when they call: for example a process that hands all of HBM to its
   own allocator at start-up, or a latency-critical loop that must not take allocator locks or
   risk an out-of-memory error mid-step. It allocates nothing: the fp32 scratch for the
   region means (2 * B * n_win^2 * C * 4 bytes) lives in a fixed 8 MiB device array inside
   the library (held by every GPU that loads it until the process exits), and a call that
   needs more returns BRA_ERR_UNSUPPORTED, with the sizes in bra_last_error_message(),
   before anything runs. One-token regions (n_win = H = W, n_win^2 <= 256) need no scratch,
   as in bra_route. The first call on each device finds that array's device address
   (cudaGetSymbolAddress), so make it before any stream capture. All calls on a device share
   the array; calls whose kernels overlap on the GPU race on it, so order them on one stream.
   The paper has no counterpart to this entry point: it is a deployment variant. */
bra_status bra_route_noalloc(const void *q, const void *k, int32_t *idx, int B, int H, int W, int C, int n_win,
                             int topk, bra_dtype dtype, void *stream);

/* Per-head routing ("医学图像分割模块：BiFormer / 双层路由注意力", §五 steps ③④): the region means
   of head h are its head_dim channels of the region means (hd = C / heads), its affinities
   A_h = hd^-1/2 qm_h km_h^T, and idx[b, h, r, :] its topk largest in the routing order above.
   q, k: device [B, H, W, C]. idx: device int32 [B, heads, n_win^2, topk], written. topk <= R
   (the pages clamp topk to R; the Python binding does, this call rejects a larger topk). Takes
   fp32 scratch for the means from the pool, like bra_route (none for one-token regions).
   BRA_ERR_UNSUPPORTED: R > 256, or a head's channels not a whole number of 16-byte vectors of
   the fp32 means (hd % 4 != 0) or, for one-token regions, of the tokens. */
bra_status bra_route_heads(const void *q, const void *k, int32_t *idx, int B, int H, int W, int C, int heads,
                           int n_win, int topk, bra_dtype dtype, void *stream);

/* Step 5 with per-head routing ("医学图像分割模块", §五 steps ⑤-⑦): head h of a query in region r
   attends over the tokens of regions idx[b, h, r, 0..topk-1]. idx: device int32
   [B, heads, n_win^2, topk] (out-of-range entries skipped and flagged, duplicates gathered as
   often as they occur); other arguments as bra_attend. bf16 with hd == 32, C % 64 == 0 and
   regions of 16, 32, 48 or 64 tokens runs on the tensor cores (BRA_ATTEND_GATHER_MMA, each head
   gathering the tiles of its own regions), everything else on CUDA cores with the routed rows
   staged in shared memory (BRA_ATTEND_SIMT); bra_set_attend_kernel may force either one, and
   forcing any other kernel makes the call BRA_ERR_UNSUPPORTED. BRA_ERR_UNSUPPORTED: hd > 128
   on CUDA cores. */
bra_status bra_attend_heads(const void *q, const void *k, const void *v, const int32_t *idx, void *out, int B,
                            int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream);

/* bra_route_heads then bra_attend_heads on one stream; the means are kept in `out` until the
   attention overwrites it, so nothing is allocated. */
bra_status bra_forward_heads(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H,
                             int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream);

/* auto_pad ("从静态到动态", §4.2: auto_pad handles the edge padding; "从零构建BiFormer", §1: a
   padding layer in front when the size is not a multiple of the region grid): the forward pass of
   an H x W map that need not be a multiple of n_win. The map is taken as padded with zeros at the
   bottom and the right to Hp x Wp, Hp = ceil(H / n_win) n_win (likewise Wp); nothing is copied:
   the kernels read zeros outside the image. The padded tokens count in the region means (a sum
   over the region divided by (Hp / n_win) (Wp / n_win)) and take part in the attention as keys
   with logit 0 and value 0; out holds the H x W queries only. q, k, v, out: device
   [B, H, W, C]; idx: device int32 [B, n_win^2, topk], written (routing of the padded map). When
   H and W are multiples of n_win this is bra_forward. Attention runs on the kernel bra_attend
   would use for the padded shape, reading the padded map through tensor maps of the true image
   (or, on CUDA cores, with guarded loads); the means use out as scratch when they fit in it,
   else the pool. */
bra_status bra_forward_auto_pad(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H,
                                int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream);

/* LePE epilogue ("医学图像分割模块", §五 step ⑧: the attention output viewed as a [C, H, W] image,
   plus its 5 x 5 depthwise convolution): y = x + bias + sum_{dy, dx} weight[c, dy, dx]
   x[b, i + dy - 2, j + dx - 2, c], zeros outside the image (nn.Conv2d(C, C, 5, padding=2,
   groups=C), cross-correlation). x, y: device [B, H, W, C] of dtype, distinct; weight: device
   fp32 [C, 5, 5]; bias: device fp32 [C]. Arithmetic in fp32, y rounded to dtype.
   BRA_ERR_INVALID_ARG also when x == y or C is not a whole number of 16-byte vectors. */
bra_status bra_lepe(const void *x, const float *weight, const float *bias, void *y, int B, int H, int W, int C,
                    bra_dtype dtype, void *stream);

/* bra_forward into `attn`, then bra_lepe(attn) into `out` (both caller-owned [B, H, W, C] of dtype,
   distinct): out = attn + lepe(attn). The epilogue reads attn right after the attention wrote it,
   while it is in L2. */
bra_status bra_forward_lepe(const void *q, const void *k, const void *v, int32_t *idx, void *attn, void *out,
                            const float *weight, const float *bias, int B, int H, int W, int C, int heads, int n_win,
                            int topk, bra_dtype dtype, void *stream);

/* Backward of step 5 with the routing index held fixed (the pages train the model, "从静态到动态",
   §3.2; top-k passes no gradient): given dout = dL/dout, the gradients of L = sum(dout * out)
   with respect to q, k and v. q, k, v, dout: device [B, H, W, C] of dtype; idx: device int32
   [B, n_win^2, topk] (out-of-range entries skipped and flagged); dq, dk, dv: device fp32
   [B, H, W, C], written (dk and dv are cleared first, then accumulated with atomics, so their
   last bits may differ between runs). bf16 with 64-token regions and 32-channel heads runs on the
   tensor cores (the bf16 inputs as they are, p and ds as two bf16 terms each: about 16
   significant bits, products exact, fp32 sums); everything else on CUDA cores in fp32.
   BRA_ERR_UNSUPPORTED: hd % 8 != 0, hd > 128, or a region of more than 256 tokens. */
bra_status bra_attend_backward(const void *q, const void *k, const void *v, const int32_t *idx, const void *dout,
                               float *dq, float *dk, float *dv, int B, int H, int W, int C, int heads, int n_win,
                               int topk, bra_dtype dtype, void *stream);

/* bra_forward on HOST buffers: copies q, k, v (host, [B, H, W, C]) to device scratch from
   the library's pool, runs the forward pass on `stream`, copies idx and out back to the
   host buffers and synchronises `stream` before returning. Page-locked host memory gives
   asynchronous, full-speed copies; pageable memory works too. */
bra_status bra_forward_host(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B,
                            int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype,
                            void *stream);

/* Force (or, with AUTO, release) one attention kernel for later calls in this process.
   Returns BRA_ERR_INVALID_ARG for an unknown value. */
bra_status bra_set_attend_kernel(bra_attend_kernel kernel);

/* Caps the grid of the persistent attention kernels (the tcgen05 and the mma.sync gather
   kernels, which split the work items of a call evenly over at most two CTAs per SM) at
   max_ctas CTAs for later calls in this process; 0 removes the cap. A small cap gives each
   CTA many consecutive work items, which tests use to exercise the carried state between
   items on small inputs. The result does not depend on it. Returns BRA_ERR_INVALID_ARG for
   max_ctas < 0. */
bra_status bra_set_max_ctas(int max_ctas);

/* The attention kernel a call with these arguments would use (after any forcing), or -1 if
   the call would be rejected or unsupported. */
int bra_selected_attend_kernel(int B, int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype);

/* A check of the bounded wait that every pipelined kernel of the library uses: launches one
   thread that waits on an mbarrier nothing ever completes, with that wait given a limit of
   limit_us microseconds (1 .. 1000000; the kernels of the forward pass use 2 s). The wait gives
   up, sets BRA_ERR_TIMEOUT in the device error word and the kernel returns, with nothing else
   in flight; bra_check_device_error then returns BRA_ERR_TIMEOUT. Computes nothing. */
bra_status bra_selftest_wait_timeout(unsigned limit_us, void *stream);

/* Synchronises `stream`, then reads and clears the current device's sticky error word:
   BRA_OK, BRA_ERR_INDEX (an idx entry outside [0, R) was skipped) or BRA_ERR_TIMEOUT. */
bra_status bra_check_device_error(void *stream);

/* Bytes of scratch bra_route / bra_forward take from the pool for these sizes (fp32 means; 0 when
   every region is one token and R <= 256, where routing reads q and k directly). */
size_t bra_route_scratch_bytes(int B, int H, int W, int C, int n_win);

/* Number of library kernels one call of `entry_point` ("bra_route", "bra_attend",
   "bra_forward", "bra_forward_host") launches with these arguments, for launch accounting
   (memset and copy nodes not counted); 0 for a call that would launch nothing or be rejected. */
int bra_kernels_per_call(const char *entry_point, int B, int H, int W, int C, int heads, int n_win, int topk,
                         bra_dtype dtype);

/* Static strings: the name of a status, and the last CUDA error message of this thread. */
const char *bra_status_string(bra_status status);
const char *bra_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* BRA_H */
