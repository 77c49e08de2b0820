// bra_api.cu -- the C ABI of libbra.so (declared in include/bra.h): argument validation,
// kernel selection, TMA descriptors, the per-device scratch pool and the device error word.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "bra.h"
#include "bra_launch.h"

namespace {

// Sticky device error word (kErrIndex | kErrTimeout), one per device.
__device__ unsigned g_device_error;

constexpr int kMaxDevices = 64;

struct DeviceState {
    std::atomic<bool> ready{false};  // set (release) after every other field
    unsigned *error_word = nullptr;
    cudaMemPool_t pool = nullptr;
    int num_sms = 0;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;  // host-copy streams of bra_forward_host
};

std::mutex g_mutex;
DeviceState g_devices[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_forced_kernel{BRA_ATTEND_AUTO};
std::atomic<int> g_max_ctas{0};
thread_local std::string g_last_error;

bra_status cuda_fail(cudaError_t e, const char *what)
{
    g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
    return BRA_ERR_CUDA;
}

// Per-device set-up on first use: error word address, SM count, scratch pool, TMA encoder.
bra_status device_state(DeviceState **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        g_last_error = "device ordinal out of range";
        return BRA_ERR_UNSUPPORTED;
    }
    DeviceState &st = g_devices[dev];
    if (!st.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!st.ready.load(std::memory_order_relaxed)) {
            void *p = nullptr;
            if ((e = cudaGetSymbolAddress(&p, g_device_error)) != cudaSuccess)
                return cuda_fail(e, "cudaGetSymbolAddress(error word)");
            st.error_word = static_cast<unsigned *>(p);
            if ((e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
                return cuda_fail(e, "cudaDeviceGetAttribute");
            cudaMemPoolProps props;
            std::memset(&props, 0, sizeof(props));
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if ((e = cudaMemPoolCreate(&st.pool, &props)) != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
            uint64_t keep = ~0ull;  // keep freed scratch in the pool
            if ((e = cudaMemPoolSetAttribute(st.pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess)
                return cuda_fail(e, "cudaMemPoolSetAttribute");
            if ((e = cudaStreamCreateWithFlags(&st.copy_in, cudaStreamNonBlocking)) != cudaSuccess ||
                (e = cudaStreamCreateWithFlags(&st.copy_out, cudaStreamNonBlocking)) != cudaSuccess)
                return cuda_fail(e, "cudaStreamCreateWithFlags");
            if (!g_encode) {
                void *fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
                if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
                    g_last_error = "cuTensorMapEncodeTiled not available from the driver";
                    return BRA_ERR_CUDA;
                }
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
            st.ready.store(true, std::memory_order_release);
        }
    }
    *out = &st;
    return BRA_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by every entry point (pointers are checked by the callers).
bra_status check_shape(int B, int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype,
                       bra::Geometry *g)
{
    if (dtype != BRA_F32 && dtype != BRA_BF16) return BRA_ERR_INVALID_ARG;
    if (B < 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0 || n_win <= 0 || topk <= 0) return BRA_ERR_INVALID_ARG;
    if (H % n_win != 0 || W % n_win != 0 || C % heads != 0) return BRA_ERR_INVALID_ARG;
    const long long R = (long long)n_win * n_win;
    if (topk > R) return BRA_ERR_INVALID_ARG;
    const int elem = dtype == BRA_BF16 ? 2 : 4;
    if (((long long)C * elem) % 16 != 0) return BRA_ERR_INVALID_ARG;
    if (R > bra::kMaxRegions) return BRA_ERR_UNSUPPORTED;
    if ((long long)H * W > 0x7fffffffLL / 2) return BRA_ERR_UNSUPPORTED;
    g->B = B;
    g->H = H;
    g->W = W;
    g->C = C;
    g->heads = heads;
    g->n_win = n_win;
    g->topk = topk;
    g->R = (int)R;
    g->hr = H / n_win;
    g->wr = W / n_win;
    g->rs = g->hr * g->wr;
    g->hd = C / heads;
    g->N = H * W;
    // The means kernel holds one region's row segment (wr tokens x C channels) in shared memory.
    if ((long long)g->wr * C * elem > 16LL * bra::kMaxMeansVectors) return BRA_ERR_UNSUPPORTED;
    return BRA_OK;
}

int choose_attend_kernel(const bra::Geometry &g, bra_dtype dtype)
{
    const bool bf16 = dtype == BRA_BF16;
    const bool simt_ok = g.hd <= bra::kSimtMaxHeadDim;
    const bool gather_ok = bf16 && bra::gather_mma_supports(g);
    const bool dense_ok = bf16 && bra::dense_mma_supports(g);
    const bool umma_ok = bf16 && bra::gather_umma_supports(g);
    const bool region_ok = bf16 && bra::region_mma_supports(g);
    switch (g_forced_kernel.load()) {
    case BRA_ATTEND_SIMT: return simt_ok ? BRA_ATTEND_SIMT : -1;
    case BRA_ATTEND_GATHER_MMA: return gather_ok ? BRA_ATTEND_GATHER_MMA : -1;
    case BRA_ATTEND_DENSE_MMA: return dense_ok ? BRA_ATTEND_DENSE_MMA : -1;
    case BRA_ATTEND_GATHER_UMMA: return umma_ok ? BRA_ATTEND_GATHER_UMMA : -1;
    case BRA_ATTEND_REGION_MMA: return region_ok ? BRA_ATTEND_REGION_MMA : -1;
    default: break;
    }
    // 4-token regions: tiles of 4 tokens x 4 heads over the routed keys only
    if (region_ok) return BRA_ATTEND_REGION_MMA;
    // Dense attention over the whole image wastes at most 4x the routed work here.
    if (dense_ok && 4LL * g.topk * g.rs >= g.N) return BRA_ATTEND_DENSE_MMA;
    if (umma_ok) return BRA_ATTEND_GATHER_UMMA;
    if (gather_ok) return BRA_ATTEND_GATHER_MMA;
    if (dense_ok) return BRA_ATTEND_DENSE_MMA;
    return simt_ok ? BRA_ATTEND_SIMT : -1;
}

// 4-D bf16 tensor map of a [B, H, W, C] array, 128-byte swizzle, box (64, bw, bh, 1); H, W: the
// image in memory (g.H, g.W unless the map is padded to the region grid).
bra_status encode_map(CUtensorMap *map, const void *base, const bra::Geometry &g, int bw, int bh, int H, int W)
{
    cuuint64_t dims[4] = {(cuuint64_t)g.C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)g.B};
    cuuint64_t strides[3] = {(cuuint64_t)g.C * 2, (cuuint64_t)W * g.C * 2, (cuuint64_t)H * W * g.C * 2};
    cuuint32_t box[4] = {64u, (cuuint32_t)bw, (cuuint32_t)bh, 1u};
    cuuint32_t elem_strides[4] = {1u, 1u, 1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_error = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
        return BRA_ERR_CUDA;
    }
    return BRA_OK;
}

// 5-D bf16 tensor map of a [B, H, W, C] array viewed as (channel in its 64-channel block, x, y,
// channel block, image), 128-byte swizzle, box (64, bw, bh, nblk, 1): the nblk channel blocks
// of a box land in shared memory one after the other, each as its own (bh x bw)-row tile.
bra_status encode_map_blocks(CUtensorMap *map, const void *base, const bra::Geometry &g, int bw, int bh, int nblk,
                             int H, int W)
{
    cuuint64_t dims[5] = {64u, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)(g.C / 64), (cuuint64_t)g.B};
    cuuint64_t strides[4] = {(cuuint64_t)g.C * 2, (cuuint64_t)W * g.C * 2, 128u, (cuuint64_t)H * W * g.C * 2};
    cuuint32_t box[5] = {64u, (cuuint32_t)bw, (cuuint32_t)bh, (cuuint32_t)nblk, 1u};
    cuuint32_t elem_strides[5] = {1u, 1u, 1u, 1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box,
                          elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_error = "cuTensorMapEncodeTiled (5-D) failed with CUresult " + std::to_string((int)r);
        return BRA_ERR_CUDA;
    }
    return BRA_OK;
}

// The routing step. `workspace` (may be NULL): caller memory of `ws_bytes` bytes, 16-byte
// aligned, that nothing reads until the stream passes this call; the fp32 means go there when
// they fit, else into scratch from the pool.
bra_status route_impl(const void *q, const void *k, int32_t *idx, const bra::Geometry &g, bra_dtype dtype,
                      cudaStream_t stream, void *workspace = nullptr, size_t ws_bytes = 0)
{
    DeviceState *st = nullptr;
    bra_status s = device_state(&st);
    if (s != BRA_OK) return s;
    if (g.rs == 1 && g.R <= 256) {
        // one-token regions: the means are the tokens, no scratch and no means kernel
        const cudaError_t e = bra::launch_route_topk_tokens(q, k, idx, g, dtype == BRA_BF16, stream);
        return e == cudaSuccess ? BRA_OK : cuda_fail(e, "routing kernel");
    }
    const size_t bytes = (size_t)2 * g.B * g.R * g.C * sizeof(float);
    const bool in_workspace = workspace && bytes <= ws_bytes;
    void *scratch = in_workspace ? workspace : nullptr;
    cudaError_t e = cudaSuccess;
    if (!in_workspace && (e = cudaMallocFromPoolAsync(&scratch, bytes, st->pool, stream)) != cudaSuccess)
        return cuda_fail(e, "cudaMallocFromPoolAsync(route scratch)");
    float *qm = static_cast<float *>(scratch);
    float *km = qm + (size_t)g.B * g.R * g.C;
    e = bra::launch_region_means(q, k, qm, km, g, dtype == BRA_BF16, st->num_sms, stream);
    if (e == cudaSuccess) e = bra::launch_route_topk(qm, km, idx, g, stream);
    cudaError_t f = in_workspace ? cudaSuccess : cudaFreeAsync(scratch, stream);
    if (e != cudaSuccess) return cuda_fail(e, "routing kernels");
    if (f != cudaSuccess) return cuda_fail(f, "cudaFreeAsync(route scratch)");
    return BRA_OK;
}

// inputs_ready: the kernel launched just before on `stream` is this library's routing kernel,
// which has already waited for the producers of q, k and v, so the attention kernel may read
// them before it waits for its predecessor (only idx comes from that kernel). H, W (>= 0): the
// image in memory when it is smaller than the region grid g (auto_pad); tokens outside it are
// zeros and are not stored.
bra_status attend_impl(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                       const bra::Geometry &g, bra_dtype dtype, cudaStream_t stream, bool inputs_ready = false,
                       int H = -1, int W = -1)
{
    if (H < 0) {
        H = g.H;
        W = g.W;
    }
    const int kernel = choose_attend_kernel(g, dtype);
    if (kernel < 0) return BRA_ERR_UNSUPPORTED;
    DeviceState *st = nullptr;
    bra_status s = device_state(&st);
    if (s != BRA_OK) return s;
    cudaError_t e = cudaSuccess;
    if (kernel == BRA_ATTEND_SIMT) {
        e = bra::launch_attend_staged(q, k, v, idx, out, g, H, W, false, dtype == BRA_BF16, st->error_word, stream);
    } else if (kernel == BRA_ATTEND_GATHER_UMMA) {
        CUtensorMap tq, tk, tv;
        if ((s = encode_map(&tq, q, g, g.wr, g.hr, H, W)) != BRA_OK) return s;
        if ((s = encode_map(&tk, k, g, g.wr, g.hr, H, W)) != BRA_OK) return s;
        if ((s = encode_map(&tv, v, g, g.wr, g.hr, H, W)) != BRA_OK) return s;
        e = bra::launch_attend_gather_umma(tq, tk, tv, idx, out, g, H, W, st->num_sms, st->error_word, stream);
    } else if (kernel == BRA_ATTEND_REGION_MMA) {
        CUtensorMap tq, tk, tv;
        if ((s = encode_map_blocks(&tq, q, g, g.W, g.H, 2, H, W)) != BRA_OK) return s;
        if ((s = encode_map_blocks(&tk, k, g, g.W, g.H, 2, H, W)) != BRA_OK) return s;
        if ((s = encode_map_blocks(&tv, v, g, g.W, g.H, 2, H, W)) != BRA_OK) return s;
        e = bra::launch_attend_region_mma(tq, tk, tv, idx, out, g, H, W, st->num_sms, st->error_word, inputs_ready,
                                          stream);
    } else if (kernel == BRA_ATTEND_GATHER_MMA) {
        CUtensorMap tq, tk, tv, to;
        int box[5];
        bra::gather_mma_box(g, box);
        if ((s = encode_map_blocks(&tq, q, g, box[1], box[2], box[3], H, W)) != BRA_OK) return s;
        if ((s = encode_map_blocks(&tk, k, g, box[1], box[2], box[3], H, W)) != BRA_OK) return s;
        if ((s = encode_map_blocks(&tv, v, g, box[1], box[2], box[3], H, W)) != BRA_OK) return s;
        if ((s = encode_map(&to, out, g, box[1], box[2], H, W)) != BRA_OK) return s;
        e = bra::launch_attend_gather_mma(tq, tk, tv, to, idx, out, g, H, W, st->num_sms, st->error_word, stream);
    } else {
        const int rows = bra::dense_mma_rows_per_split(g, st->num_sms);
        CUtensorMap tq, tk, tv, to;
        if ((s = encode_map(&tq, q, g, g.W, rows, H, W)) != BRA_OK) return s;
        if ((s = encode_map(&tk, k, g, g.W, g.H, H, W)) != BRA_OK) return s;
        if ((s = encode_map(&tv, v, g, g.W, g.H, H, W)) != BRA_OK) return s;
        if ((s = encode_map(&to, out, g, g.W, rows, H, W)) != BRA_OK) return s;
        e = bra::launch_attend_dense_mma(tq, tk, tv, to, idx, g, rows, st->error_word, inputs_ready, H, stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
    return BRA_OK;
}

// One-token regions that the dense kernel serves: routing runs inside it (one launch).
bool fused_forward(const bra::Geometry &g, bra_dtype dtype)
{
    return choose_attend_kernel(g, dtype) == BRA_ATTEND_DENSE_MMA && bra::route_dense_supports(g, dtype == BRA_BF16);
}

// The forward pass on device buffers: the fused kernel where it serves the shape, else the
// routing step (its fp32 means in `out`, which nothing else writes until the attention kernel)
// followed by the attention kernel.
bra_status forward_impl(const void *q, const void *k, const void *v, int32_t *idx, void *out, const bra::Geometry &g,
                        bra_dtype dtype, cudaStream_t stream)
{
    if (fused_forward(g, dtype)) {
        DeviceState *st = nullptr;
        bra_status s = device_state(&st);
        if (s != BRA_OK) return s;
        CUtensorMap tq, tk, tv, to;
        if ((s = encode_map(&tq, q, g, g.W, g.H, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&tk, k, g, g.W, g.H, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&tv, v, g, g.W, g.H, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&to, out, g, g.W, g.H, g.H, g.W)) != BRA_OK) return s;
        const cudaError_t e = bra::launch_route_attend_dense(tq, tk, tv, to, idx, g, st->error_word, stream);
        return e == cudaSuccess ? BRA_OK : cuda_fail(e, "fused routing and attention kernel");
    }
    const size_t out_bytes = (size_t)g.B * g.H * g.W * g.C * (dtype == BRA_BF16 ? 2 : 4);
    bra_status s = route_impl(q, k, idx, g, dtype, stream, out, out_bytes);
    if (s != BRA_OK) return s;
    return attend_impl(q, k, v, idx, out, g, dtype, stream, true);
}

}  // namespace

namespace bra {

void set_last_error(const std::string &msg) { g_last_error = msg; }

int persistent_grid(long long nitems, int num_sms, int per_sm)
{
    long long grid = (long long)per_sm * num_sms;
    const int cap = g_max_ctas.load();
    if (cap > 0 && grid > cap) grid = cap;
    if (grid > nitems) grid = nitems;
    return grid < 1 ? 1 : (int)grid;
}

bra_status check_route_args(const void *q, const void *k, const int32_t *idx, int B, int H, int W, int C, int n_win,
                            int topk, bra_dtype dtype, Geometry *g)
{
    bra_status s = check_shape(B, H, W, C, 1, n_win, topk, dtype, g);
    if (s != BRA_OK || B == 0) return s;
    if (!q || !k || !idx) return BRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4)) return BRA_ERR_INVALID_ARG;
    return BRA_OK;
}

}  // namespace bra

extern "C" {

bra_status bra_route(const void *q, const void *k, int32_t *idx, int B, int H, int W, int C, int n_win, int topk,
                     bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, 1, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if (!q || !k || !idx) return BRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4)) return BRA_ERR_INVALID_ARG;
    return route_impl(q, k, idx, g, dtype, static_cast<cudaStream_t>(stream));
}

bra_status bra_attend(const void *q, const void *k, const void *v, const int32_t *idx, void *out, int B, int H,
                      int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if (!q || !k || !v || !idx || !out) return BRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(idx, 4))
        return BRA_ERR_INVALID_ARG;
    return attend_impl(q, k, v, idx, out, g, dtype, static_cast<cudaStream_t>(stream));
}

bra_status bra_forward(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H, int W,
                       int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if (!q || !k || !v || !idx || !out) return BRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(idx, 4))
        return BRA_ERR_INVALID_ARG;
    if (choose_attend_kernel(g, dtype) < 0) return BRA_ERR_UNSUPPORTED;
    return forward_impl(q, k, v, idx, out, g, dtype, static_cast<cudaStream_t>(stream));
}

bra_status bra_forward_host(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H,
                            int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if (!q || !k || !v || !idx || !out) return BRA_ERR_INVALID_ARG;
    if (choose_attend_kernel(g, dtype) < 0) return BRA_ERR_UNSUPPORTED;
    DeviceState *dst = nullptr;
    if ((s = device_state(&dst)) != BRA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t elem = dtype == BRA_BF16 ? 2 : 4;
    const size_t image = (size_t)H * W * C * elem, image_idx = (size_t)g.R * topk * sizeof(int32_t);
    const size_t tensor = (size_t)B * image;
    const size_t tensor_padded = (tensor + 255) & ~(size_t)255;
    const size_t idx_bytes = (size_t)B * image_idx;
    uint8_t *buf = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&buf), 4 * tensor_padded + idx_bytes, dst->pool, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync(host staging)");
    uint8_t *dq = buf, *dk = buf + tensor_padded, *dv = buf + 2 * tensor_padded, *dout = buf + 3 * tensor_padded;
    int32_t *didx = reinterpret_cast<int32_t *>(buf + 4 * tensor_padded);
    // The batch in up to kChunks chunks of whole images: the copies in of chunk c + 1 (stream
    // copy_in) and out of chunk c - 1 (copy_out) overlap the computation of chunk c (`stream`).
    constexpr int kChunks = 4;
    const int nchunk = B < kChunks ? B : kChunks;
    cudaEvent_t ev_start = nullptr, ev_in[kChunks] = {}, ev_done[kChunks] = {}, ev_out = nullptr;
    auto make_event = [&](cudaEvent_t *ev) {
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    };
    make_event(&ev_start);
    make_event(&ev_out);
    for (int c = 0; c < nchunk; ++c) {
        make_event(&ev_in[c]);
        make_event(&ev_done[c]);
    }
    // the staging buffer exists from here on `stream`; the copy streams start after it
    if (e == cudaSuccess) e = cudaEventRecord(ev_start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(dst->copy_in, ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(dst->copy_out, ev_start, 0);
    int b0 = 0;
    for (int c = 0; c < nchunk && e == cudaSuccess && s == BRA_OK; ++c) {
        const int nb = B / nchunk + (c < B % nchunk ? 1 : 0);
        const size_t off = (size_t)b0 * image, bytes = (size_t)nb * image;
        const size_t ioff = (size_t)b0 * image_idx / sizeof(int32_t), ibytes = (size_t)nb * image_idx;
        const uint8_t *hq = static_cast<const uint8_t *>(q), *hk = static_cast<const uint8_t *>(k);
        const uint8_t *hv = static_cast<const uint8_t *>(v);
        e = cudaMemcpyAsync(dq + off, hq + off, bytes, cudaMemcpyHostToDevice, dst->copy_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(dk + off, hk + off, bytes, cudaMemcpyHostToDevice, dst->copy_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(dv + off, hv + off, bytes, cudaMemcpyHostToDevice, dst->copy_in);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[c], dst->copy_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_in[c], 0);
        if (e != cudaSuccess) break;
        bra::Geometry gc = g;
        gc.B = nb;
        s = forward_impl(dq + off, dk + off, dv + off, didx + ioff, dout + off, gc, dtype, st);
        if (s != BRA_OK) break;
        e = cudaEventRecord(ev_done[c], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(dst->copy_out, ev_done[c], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<uint8_t *>(out) + off, dout + off, bytes, cudaMemcpyDeviceToHost,
                                dst->copy_out);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(idx + ioff, didx + ioff, ibytes, cudaMemcpyDeviceToHost, dst->copy_out);
        b0 += nb;
    }
    // `stream` resumes after the last copy out; the buffer goes back to the pool then. After an
    // error the host waits for both copy streams first, so that no copy still uses the buffer.
    cudaError_t j = ev_out ? cudaEventRecord(ev_out, dst->copy_out) : cudaErrorInvalidValue;
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, ev_out, 0);
    if (j != cudaSuccess || e != cudaSuccess || s != BRA_OK) {
        cudaStreamSynchronize(dst->copy_in);
        cudaStreamSynchronize(dst->copy_out);
    }
    cudaError_t f = cudaFreeAsync(buf, st);
    cudaError_t y = cudaStreamSynchronize(st);
    for (cudaEvent_t ev : {ev_start, ev_out})
        if (ev) cudaEventDestroy(ev);
    for (int c = 0; c < nchunk; ++c) {
        if (ev_in[c]) cudaEventDestroy(ev_in[c]);
        if (ev_done[c]) cudaEventDestroy(ev_done[c]);
    }
    if (s != BRA_OK) return s;
    if (e != cudaSuccess) return cuda_fail(e, "host copies");
    if (j != cudaSuccess) return cuda_fail(j, "copy stream join");
    if (f != cudaSuccess) return cuda_fail(f, "cudaFreeAsync(host staging)");
    if (y != cudaSuccess) return cuda_fail(y, "cudaStreamSynchronize");
    return BRA_OK;
}

// ---------------------------------------------------------------- per-head routing

static bra_status route_heads_impl(const void *q, const void *k, int32_t *idx, const bra::Geometry &g,
                                   bra_dtype dtype, cudaStream_t stream, void *workspace = nullptr,
                                   size_t ws_bytes = 0)
{
    DeviceState *st = nullptr;
    bra_status s = device_state(&st);
    if (s != BRA_OK) return s;
    const bool bf16 = dtype == BRA_BF16;
    if (g.rs == 1) {  // one-token regions: the means are the tokens
        const cudaError_t e = bra::launch_route_heads_tokens(q, k, idx, g, bf16, stream);
        return e == cudaSuccess ? BRA_OK : cuda_fail(e, "per-head routing kernel");
    }
    const size_t bytes = (size_t)2 * g.B * g.R * g.C * sizeof(float);
    const bool in_workspace = workspace && bytes <= ws_bytes;
    void *scratch = in_workspace ? workspace : nullptr;
    cudaError_t e = cudaSuccess;
    if (!in_workspace && (e = cudaMallocFromPoolAsync(&scratch, bytes, st->pool, stream)) != cudaSuccess)
        return cuda_fail(e, "cudaMallocFromPoolAsync(route scratch)");
    float *qm = static_cast<float *>(scratch);
    float *km = qm + (size_t)g.B * g.R * g.C;
    e = bra::launch_region_means(q, k, qm, km, g, bf16, st->num_sms, stream);
    if (e == cudaSuccess) e = bra::launch_route_heads(qm, km, idx, g, stream);
    cudaError_t f = in_workspace ? cudaSuccess : cudaFreeAsync(scratch, stream);
    if (e != cudaSuccess) return cuda_fail(e, "per-head routing kernels");
    if (f != cudaSuccess) return cuda_fail(f, "cudaFreeAsync(route scratch)");
    return BRA_OK;
}

// The attention kernel of per-head routing: the mma.sync gather kernel (bf16, hd == 32, rs % 16
// == 0, rs <= 64) in its per-head mode; for small images with few tokens per region the dense
// kernel with one routing-count plane per head (under the same rule as the shared index);
// else the CUDA-core kernel. A forced kernel that does not take per-head indices (or cannot
// serve the shape) makes the call unsupported.
static int choose_heads_kernel(const bra::Geometry &g, bra_dtype dtype)
{
    const bool simt_ok = g.hd <= bra::kSimtMaxHeadDim;
    const bool gather_ok = dtype == BRA_BF16 && bra::gather_mma_supports(g);
    const bool dense_ok = dtype == BRA_BF16 && bra::dense_mma_supports(g);
    switch (g_forced_kernel.load()) {
    case BRA_ATTEND_AUTO:
        if (gather_ok) return BRA_ATTEND_GATHER_MMA;
        if (dense_ok && 4LL * g.topk * g.rs >= g.N) return BRA_ATTEND_DENSE_MMA;
        return simt_ok ? BRA_ATTEND_SIMT : -1;
    case BRA_ATTEND_SIMT: return simt_ok ? BRA_ATTEND_SIMT : -1;
    case BRA_ATTEND_GATHER_MMA: return gather_ok ? BRA_ATTEND_GATHER_MMA : -1;
    case BRA_ATTEND_DENSE_MMA: return dense_ok ? BRA_ATTEND_DENSE_MMA : -1;
    default: return -1;
    }
}

static bra_status attend_heads_impl(const void *q, const void *k, const void *v, const int32_t *idx, void *out,
                                    const bra::Geometry &g, bra_dtype dtype, cudaStream_t stream)
{
    const int kernel = choose_heads_kernel(g, dtype);
    if (kernel < 0) return BRA_ERR_UNSUPPORTED;
    DeviceState *st = nullptr;
    bra_status s = device_state(&st);
    if (s != BRA_OK) return s;
    cudaError_t e = cudaSuccess;
    if (kernel == BRA_ATTEND_SIMT) {
        e = bra::launch_attend_staged(q, k, v, idx, out, g, g.H, g.W, true, dtype == BRA_BF16, st->error_word, stream);
    } else if (kernel == BRA_ATTEND_DENSE_MMA) {
        const int rows = bra::dense_mma_rows_per_split(g, st->num_sms);
        CUtensorMap tq, tk, tv, to;
        if ((s = encode_map(&tq, q, g, g.W, rows, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&tk, k, g, g.W, g.H, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&tv, v, g, g.W, g.H, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&to, out, g, g.W, rows, g.H, g.W)) != BRA_OK) return s;
        e = bra::launch_attend_dense_mma(tq, tk, tv, to, idx, g, rows, st->error_word, false, g.H, stream, true);
    } else {
        // q: the item's NCB blocks in one box; k, v: one block per box (each head its own region)
        CUtensorMap tq, tk, tv, to;
        int box[5];
        bra::gather_mma_box(g, box);
        if ((s = encode_map_blocks(&tq, q, g, box[1], box[2], box[3], g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map_blocks(&tk, k, g, box[1], box[2], 1, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map_blocks(&tv, v, g, box[1], box[2], 1, g.H, g.W)) != BRA_OK) return s;
        if ((s = encode_map(&to, out, g, box[1], box[2], g.H, g.W)) != BRA_OK) return s;
        e = bra::launch_attend_gather_mma(tq, tk, tv, to, idx, out, g, g.H, g.W, st->num_sms, st->error_word, stream,
                                          true);
    }
    return e == cudaSuccess ? BRA_OK : cuda_fail(e, "per-head attention kernel");
}

static bra_status check_data_ptrs(const void *q, const void *k, const void *v, const int32_t *idx, const void *out)
{
    if (!q || !k || !v || !idx || !out) return BRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(idx, 4))
        return BRA_ERR_INVALID_ARG;
    return BRA_OK;
}

bra_status bra_route_heads(const void *q, const void *k, int32_t *idx, int B, int H, int W, int C, int heads,
                           int n_win, int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if (!q || !k || !idx) return BRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4)) return BRA_ERR_INVALID_ARG;
    if (!bra::route_heads_supports(g, dtype == BRA_BF16)) return BRA_ERR_UNSUPPORTED;
    return route_heads_impl(q, k, idx, g, dtype, static_cast<cudaStream_t>(stream));
}

bra_status bra_attend_heads(const void *q, const void *k, const void *v, const int32_t *idx, void *out, int B,
                            int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if ((s = check_data_ptrs(q, k, v, idx, out)) != BRA_OK) return s;
    return attend_heads_impl(q, k, v, idx, out, g, dtype, static_cast<cudaStream_t>(stream));
}

bra_status bra_forward_heads(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H,
                             int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if ((s = check_data_ptrs(q, k, v, idx, out)) != BRA_OK) return s;
    if (!bra::route_heads_supports(g, dtype == BRA_BF16) || choose_heads_kernel(g, dtype) < 0)
        return BRA_ERR_UNSUPPORTED;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t out_bytes = (size_t)B * H * W * C * (dtype == BRA_BF16 ? 2 : 4);
    if ((s = route_heads_impl(q, k, idx, g, dtype, cs, out, out_bytes)) != BRA_OK) return s;
    return attend_heads_impl(q, k, v, idx, out, g, dtype, cs);
}

// ---------------------------------------------------------------- auto_pad

bra_status bra_forward_auto_pad(const void *q, const void *k, const void *v, int32_t *idx, void *out, int B, int H,
                                int W, int C, int heads, int n_win, int topk, bra_dtype dtype, void *stream)
{
    if (H <= 0 || W <= 0 || n_win <= 0) return BRA_ERR_INVALID_ARG;
    if (H % n_win == 0 && W % n_win == 0)  // nothing to pad: the ordinary forward pass
        return bra_forward(q, k, v, idx, out, B, H, W, C, heads, n_win, topk, dtype, stream);
    const long long Hp = (long long)(H + n_win - 1) / n_win * n_win, Wp = (long long)(W + n_win - 1) / n_win * n_win;
    if (Hp > 0x7fffffffLL || Wp > 0x7fffffffLL) return BRA_ERR_UNSUPPORTED;
    bra::Geometry g;  // the padded region grid
    bra_status s = check_shape(B, (int)Hp, (int)Wp, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if ((s = check_data_ptrs(q, k, v, idx, out)) != BRA_OK) return s;
    if (choose_attend_kernel(g, dtype) < 0) return BRA_ERR_UNSUPPORTED;
    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != BRA_OK) return s;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == BRA_BF16;
    // the fp32 means in out when they fit (it is written only by the attention), else pool scratch
    const size_t bytes = (size_t)2 * g.B * g.R * g.C * sizeof(float);
    const size_t out_bytes = (size_t)B * H * W * C * (bf16 ? 2 : 4);
    const bool in_out = bytes <= out_bytes;
    void *scratch = in_out ? out : nullptr;
    cudaError_t e = cudaSuccess;
    if (!in_out && (e = cudaMallocFromPoolAsync(&scratch, bytes, st->pool, cs)) != cudaSuccess)
        return cuda_fail(e, "cudaMallocFromPoolAsync(route scratch)");
    float *qm = static_cast<float *>(scratch);
    float *km = qm + (size_t)g.B * g.R * g.C;
    e = bra::launch_region_means_padded(q, k, qm, km, g, H, W, bf16, cs);
    if (e == cudaSuccess) e = bra::launch_route_topk(qm, km, idx, g, cs);
    cudaError_t f = in_out ? cudaSuccess : cudaFreeAsync(scratch, cs);
    if (e != cudaSuccess) return cuda_fail(e, "auto_pad routing kernels");
    if (f != cudaSuccess) return cuda_fail(f, "cudaFreeAsync(route scratch)");
    // the attention kernels read the padded grid through maps of the H x W image (zeros beyond it)
    return attend_impl(q, k, v, idx, out, g, dtype, cs, true, H, W);
}

// ---------------------------------------------------------------- LePE

bra_status bra_lepe(const void *x, const float *weight, const float *bias, void *y, int B, int H, int W, int C,
                    bra_dtype dtype, void *stream)
{
    if (dtype != BRA_F32 && dtype != BRA_BF16) return BRA_ERR_INVALID_ARG;
    if (B < 0 || H <= 0 || W <= 0 || C <= 0) return BRA_ERR_INVALID_ARG;
    if (!bra::lepe_supports(C, dtype == BRA_BF16)) return BRA_ERR_INVALID_ARG;
    if (B == 0) return BRA_OK;
    if (!x || !weight || !bias || !y || x == y) return BRA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(weight, 4) || !aligned(bias, 4)) return BRA_ERR_INVALID_ARG;
    if ((long long)B * H * W > 0x7fffffffLL) return BRA_ERR_UNSUPPORTED;
    const cudaError_t e = bra::launch_lepe(x, weight, bias, y, B, H, W, C, dtype == BRA_BF16,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BRA_OK : cuda_fail(e, "LePE kernel");
}

bra_status bra_forward_lepe(const void *q, const void *k, const void *v, int32_t *idx, void *attn, void *out,
                            const float *weight, const float *bias, int B, int H, int W, int C, int heads, int n_win,
                            int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if (!out || !weight || !bias || !aligned(out, 16) || !aligned(weight, 4) || !aligned(bias, 4) || out == attn)
        return BRA_ERR_INVALID_ARG;
    if ((s = bra_forward(q, k, v, idx, attn, B, H, W, C, heads, n_win, topk, dtype, stream)) != BRA_OK) return s;
    return bra_lepe(attn, weight, bias, out, B, H, W, C, dtype, stream);
}

// ---------------------------------------------------------------- backward

bra_status bra_attend_backward(const void *q, const void *k, const void *v, const int32_t *idx, const void *dout,
                               float *dq, float *dk, float *dv, int B, int H, int W, int C, int heads, int n_win,
                               int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = check_shape(B, H, W, C, heads, n_win, topk, dtype, &g);
    if (s != BRA_OK) return s;
    if (B == 0) return BRA_OK;
    if ((s = check_data_ptrs(q, k, v, idx, dout)) != BRA_OK) return s;
    if (!dq || !dk || !dv || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16)) return BRA_ERR_INVALID_ARG;
    if (!bra::attend_backward_supports(g)) return BRA_ERR_UNSUPPORTED;
    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != BRA_OK) return s;
    const cudaError_t e = bra::launch_attend_backward(q, k, v, idx, dout, dq, dk, dv, g, dtype == BRA_BF16,
                                                      st->error_word, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BRA_OK : cuda_fail(e, "backward kernel");
}

bra_status bra_selftest_wait_timeout(unsigned limit_us, void *stream)
{
    if (limit_us == 0 || limit_us > 1000000u) return BRA_ERR_INVALID_ARG;
    DeviceState *st = nullptr;
    bra_status s = device_state(&st);
    if (s != BRA_OK) return s;
    const cudaError_t e =
        bra::launch_wait_timeout(st->error_word, 1000ull * limit_us, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BRA_OK : cuda_fail(e, "wait self-test kernel");
}

bra_status bra_set_attend_kernel(bra_attend_kernel kernel)
{
    if (kernel < BRA_ATTEND_AUTO || kernel > BRA_ATTEND_REGION_MMA) return BRA_ERR_INVALID_ARG;
    g_forced_kernel.store(kernel);
    return BRA_OK;
}

bra_status bra_set_max_ctas(int max_ctas)
{
    if (max_ctas < 0) return BRA_ERR_INVALID_ARG;
    g_max_ctas.store(max_ctas);
    return BRA_OK;
}

int bra_selected_attend_kernel(int B, int H, int W, int C, int heads, int n_win, int topk, bra_dtype dtype)
{
    bra::Geometry g;
    if (check_shape(B, H, W, C, heads, n_win, topk, dtype, &g) != BRA_OK) return -1;
    return choose_attend_kernel(g, dtype);
}

bra_status bra_check_device_error(void *stream)
{
    DeviceState *st = nullptr;
    bra_status s = device_state(&st);
    if (s != BRA_OK) return s;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned word = 0;
    if ((e = cudaMemcpy(&word, st->error_word, sizeof(word), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "read error word");
    if ((e = cudaMemset(st->error_word, 0, sizeof(word))) != cudaSuccess) return cuda_fail(e, "clear error word");
    if (word & bra::kErrTimeout) return BRA_ERR_TIMEOUT;
    if (word & bra::kErrIndex) return BRA_ERR_INDEX;
    return BRA_OK;
}

size_t bra_route_scratch_bytes(int B, int H, int W, int C, int n_win)
{
    if (B <= 0 || H <= 0 || W <= 0 || C <= 0 || n_win <= 0) return 0;
    if (H == n_win && W == n_win && n_win * n_win <= 256) return 0;  // one-token regions: no means
    return (size_t)2 * B * n_win * n_win * C * sizeof(float);
}

int bra_kernels_per_call(const char *entry_point, int B, int H, int W, int C, int heads, int n_win, int topk,
                         bra_dtype dtype)
{
    if (!entry_point || B <= 0) return 0;
    bra::Geometry g;
    if (check_shape(B, H, W, C, heads, n_win, topk, dtype, &g) != BRA_OK) return 0;
    const int route = (g.rs == 1 && g.R <= 256) ? 1 : 2;
    const int attend = choose_attend_kernel(g, dtype) < 0 ? 0 : 1;
    if (!std::strcmp(entry_point, "bra_route")) return route;
    if (!std::strcmp(entry_point, "bra_attend")) return attend;
    if (!std::strcmp(entry_point, "bra_forward") || !std::strcmp(entry_point, "bra_forward_host"))
        return attend ? (fused_forward(g, dtype) ? 1 : route + attend) : 0;
    return 0;
}

const char *bra_status_string(bra_status status)
{
    switch (status) {
    case BRA_OK: return "BRA_OK";
    case BRA_ERR_INVALID_ARG: return "BRA_ERR_INVALID_ARG";
    case BRA_ERR_UNSUPPORTED: return "BRA_ERR_UNSUPPORTED";
    case BRA_ERR_CUDA: return "BRA_ERR_CUDA";
    case BRA_ERR_INDEX: return "BRA_ERR_INDEX";
    case BRA_ERR_TIMEOUT: return "BRA_ERR_TIMEOUT";
    default: return "BRA_ERR_UNKNOWN";
    }
}

const char *bra_last_error_message(void) { return g_last_error.c_str(); }

}  // extern "C"
