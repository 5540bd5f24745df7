// stream_gemv.cu -- the streamed decode GEMV over block-quantised weights
// (dense Q4/Q8 and grouped routed-expert Q4), sm_100a.
//
// The decode step is a GEMV per quantisation format with the dequantisation
// inside the inner loop (BaseRT, gist.science technical summary,
// "Methodologie" -> "Kernel Fusie en Specialisatie"), and it is bound by
// memory bandwidth ("De 'Big Model' Realiteit"; the follow-up paper's
// results paragraph says the same of its decode path).  So the design goal
// here is one thing: keep HBM busy with the packed weight bytes and read each
// of them exactly once.
//
// Work decomposition (stream-K over chunks).  A matrix is cut into bands of
// 16 rows, a band into chunks of 256 weights along K; chunks are numbered
// band-major (all chunks of band 0, then band 1, ...).  Every warp of the grid
// is an independent worker that takes one contiguous range of that numbering
// (ranges differ by at most one chunk, so every SM streams the same number of
// bytes whatever the matrix shape).  A worker owns a ring of shared-memory
// slots and its own mbarriers; its lane 0 keeps `stages - 1` chunks of TMA
// loads in flight ahead of the chunk the warp is computing.
//
// A band that lies wholly inside one worker's range is written straight to y.
// A band cut by range boundaries is summed deterministically: each worker that
// touched it stores its fp32 partial (16 rows x 8 columns) in the workspace and
// bumps the band's arrival counter; the last to arrive adds the partials in
// worker order, writes y and resets the counter to zero.  No worker ever waits
// for another.
//
// Routed experts: every CTA sorts the (token, slot) -> expert list (at most 64
// entries) in shared memory, which gives the same grouping on every CTA
// without a separate kernel.  Each distinct expert (split into pieces of at
// most 8 routed slots, the mma's N) becomes one "matrix" of the stream-K
// numbering, so each routed expert's weights are read once and multiplied
// with all of its tokens.  Per-slot outputs are written directly; the
// routing-weighted combine runs as a second small kernel in slot order.
#include <cuda_fp16.h>

#include <cstring>

#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {

constexpr int kMaxSlots = 64;   // B * topk

struct GemvArgs {
    CUtensorMap tm_codes;
    CUtensorMap tm_scales;
    const __half *x;
    float *out;         // dense: y [B][N]; experts: per-slot [B*topk][N]
    int N, K, B;
    int cpb;            // chunks per band
    int nbands;         // bands per matrix (or per expert piece)
    int wmax;           // gridDim.x * kWarps
    int *counters;      // one per (piece, band), zero on entry and exit
    float *partials;    // [wmax][2][128]
    int *status;        // device status word or null
    // routed experts
    int E, topk, x_per_slot;
    const int *idx;
};

struct ExpertGroups {
    int npieces;
    int nvalid;
    int piece_expert[kMaxSlots];
    int piece_first[kMaxSlots];
    int piece_count[kMaxSlots];
    int sorted_slot[kMaxSlots];     // slot id b*topk + s, sorted by (expert, slot)
    int key[kMaxSlots];
};

// Sort the routed slots by (expert, slot) and cut them into pieces of at most
// 8 slots of one expert.  Run by warp 0; invalid indices are left out.
__device__ void group_experts(const GemvArgs &a, ExpertGroups &grp)
{
    const int lane = threadIdx.x & 31;
    const int M = a.B * a.topk;
    for (int i = lane; i < M; i += 32) {
        const int e = a.idx[i];
        grp.key[i] = (e >= 0 && e < a.E) ? e * kMaxSlots + i : 0x7fffffff;
    }
    __syncwarp();
    int nvalid = 0;
    for (int i = lane; i < M; i += 32) {
        const int ki = grp.key[i];
        int r = 0;
        for (int j = 0; j < M; j++)
            r += grp.key[j] < ki;
        if (ki != 0x7fffffff)
            grp.sorted_slot[r] = i;
    }
    for (int j = 0; j < M; j++)
        nvalid += grp.key[j] != 0x7fffffff;
    __syncwarp();
    if (lane == 0) {
        int np = 0, cur = -1;
        for (int r = 0; r < nvalid; r++) {
            const int e = grp.key[grp.sorted_slot[r]] / kMaxSlots;
            if (e != cur || grp.piece_count[np - 1] == 8) {
                grp.piece_expert[np] = e;
                grp.piece_first[np] = r;
                grp.piece_count[np] = 0;
                np++;
                cur = e;
            }
            grp.piece_count[np - 1]++;
        }
        grp.npieces = np;
        grp.nvalid = nvalid;
    }
    __syncwarp();
}

// Index of the worker whose range holds chunk c (ranges: [w*T/W, (w+1)*T/W)).
__device__ __forceinline__ long long worker_of(long long c, long long T, long long W)
{
    return ((c + 1) * W - 1) / T;
}
__device__ __forceinline__ long long range_start(long long w, long long T, long long W)
{
    return w * T / W;
}

template <int FMT, bool MOE>
__global__ void __launch_bounds__(kThreads, 2) stream_gemv_kernel(const __grid_constant__ GemvArgs a)
{
    constexpr int D = Fmt<FMT>::kStages;
    constexpr int CB = Fmt<FMT>::kCodeBytes;
    constexpr uint32_t kTx = CB + kScaleBytes;

    extern __shared__ uint8_t smem_raw[];
    __shared__ ExpertGroups grp;

    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t codes_ring = base + (uint32_t)(warp * D * CB);
    const uint32_t scales_ring = base + (uint32_t)(kWarps * D * CB + warp * D * kScaleBytes);
    const uint32_t bars = base + (uint32_t)(kWarps * D * (CB + kScaleBytes) + warp * D * 8);

    pdl_launch_dependents();
    // Everything below reads x / idx or writes the outputs and the workspace,
    // so it waits for the previous kernel on the stream.
    pdl_wait();

    long long units = 1;
    if constexpr (MOE) {
        if (warp == 0)
            group_experts(a, grp);
        __syncthreads();
        units = grp.npieces;
        // CTA 0 reports invalid indices and zeroes their per-slot outputs.
        if (blockIdx.x == 0 && grp.nvalid < a.B * a.topk) {
            if (threadIdx.x == 0 && a.status)
                atomicOr(a.status, kStatusExpertIndex);
            if (a.out) {
                for (int i = 0; i < a.B * a.topk; i++) {
                    if (grp.key[i] != 0x7fffffff)
                        continue;
                    for (int r = threadIdx.x; r < a.N; r += kThreads)
                        a.out[(size_t)i * a.N + r] = 0.f;
                }
            }
        }
    }

    const long long bands_total = units * a.nbands;
    const long long T = bands_total * a.cpb;
    const long long W = T < a.wmax ? T : a.wmax;
    const long long w = (long long)warp * gridDim.x + blockIdx.x;
    if (w >= W)
        return;

    if (lane == 0) {
        for (int s = 0; s < D; s++)
            mbar_init(bars + 8 * s, 1);
        fence_barrier_init();
        prefetch_tensormap(&a.tm_codes);
        prefetch_tensormap(&a.tm_scales);
    }
    __syncwarp();

    const long long c0 = range_start(w, T, W);
    const long long c1 = range_start(w + 1, T, W);
    const int n = (int)(c1 - c0);
    const uint64_t pol = policy_evict_first();
    const int nb32 = a.K / kBlock;

    auto issue = [&](int i) {
        if (lane != 0)
            return;
        const long long c = c0 + i;
        const long long gb = c / a.cpb;
        const int kp = (int)(c - gb * a.cpb);
        const int unit = (int)(gb / a.nbands);
        const int row = (int)(gb - (long long)unit * a.nbands) * kChunkRows;
        const int slot = i % D;
        const uint32_t bar = bars + 8 * slot;
        const uint32_t cdst = codes_ring + (uint32_t)(slot * CB);
        const uint32_t sdst = scales_ring + (uint32_t)(slot * kScaleBytes);
        mbar_arrive_expect_tx(bar, kTx);
        if constexpr (MOE) {
            const int e = grp.piece_expert[unit];
            tma_load_3d(cdst, &a.tm_codes, bar, kp * 128, row, e, pol);
            tma_load_3d(sdst, &a.tm_scales, bar, kp * 8, row, e, pol);
        } else {
#pragma unroll
            for (int bx = 0; bx < Fmt<FMT>::kBoxes; bx++)
                tma_load_2d(cdst + bx * kBoxBytes, &a.tm_codes, bar,
                            kp * 128 * Fmt<FMT>::kBoxes + bx * 128, row, pol);
            tma_load_2d(sdst, &a.tm_scales, bar, kp * 8, row, pol);
        }
    };

    // Output of one band: acc holds (row g, col 2t), (row g, col 2t+1),
    // (row g+8, col 2t), (row g+8, col 2t+1).
    auto store_band = [&](long long gb, const float (&v)[4]) {
        const int unit = (int)(gb / a.nbands);
        const int r0 = (int)(gb - (long long)unit * a.nbands) * kChunkRows + g;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const int row = r0 + ((q & 2) ? 8 : 0);
            const int col = 2 * t + (q & 1);
            if (row >= a.N)
                continue;
            if constexpr (MOE) {
                if (col < grp.piece_count[unit]) {
                    const int slot = grp.sorted_slot[grp.piece_first[unit] + col];
                    a.out[(size_t)slot * a.N + row] = v[q];
                }
            } else {
                if (col < a.B)
                    a.out[(size_t)col * a.N + row] = v[q];
            }
        }
    };

    auto flush = [&](long long gb, const float (&acc)[4]) {
        const long long bs = gb * a.cpb, be = bs + a.cpb;
        if (bs >= c0 && be <= c1) {
            store_band(gb, acc);
            return;
        }
        const int myslot = (gb == c0 / a.cpb) ? 0 : 1;
        float4 *mine = reinterpret_cast<float4 *>(a.partials) + ((size_t)w * 2 + myslot) * 32 + lane;
        __stcg(mine, make_float4(acc[0], acc[1], acc[2], acc[3]));
        __threadfence();
        __syncwarp();
        const long long wf = worker_of(bs, T, W), wl = worker_of(be - 1, T, W);
        int old = 0;
        if (lane == 0)
            old = atomicAdd(&a.counters[gb], 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != (int)(wl - wf))
            return;
        __threadfence();
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        for (long long v = wf; v <= wl; v++) {
            float4 p;
            if (v == w) {
                p = make_float4(acc[0], acc[1], acc[2], acc[3]);
            } else {
                const int sl = (gb == range_start(v, T, W) / a.cpb) ? 0 : 1;
                p = __ldcg(reinterpret_cast<const float4 *>(a.partials) + ((size_t)v * 2 + sl) * 32 + lane);
            }
            s[0] += p.x;
            s[1] += p.y;
            s[2] += p.z;
            s[3] += p.w;
        }
        store_band(gb, s);
        if (lane == 0)
            a.counters[gb] = 0;
    };

    // Prologue: fill the ring.
    const int pre = n < D - 1 ? n : D - 1;
    for (int i = 0; i < pre; i++)
        issue(i);

    long long cur = -1;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const __half *xrow = nullptr;
    if constexpr (!MOE)
        xrow = (g < a.B) ? a.x + (size_t)g * a.K : nullptr;

    int i = 0;
    for (; i < n; i++) {
        if (i + D - 1 < n) {
            __syncwarp();
            issue(i + D - 1);
        }
        const int slot = i % D;
        if (!mbar_wait_bounded(bars + 8 * slot, (uint32_t)((i / D) & 1))) {
            if (lane == 0 && a.status)
                atomicOr(a.status, kStatusTimeout);
            break;
        }
        const long long c = c0 + i;
        const long long gb = c / a.cpb;
        const int kp = (int)(c - gb * a.cpb);
        if (gb != cur) {
            if (cur >= 0)
                flush(cur, acc);
            cur = gb;
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            if constexpr (MOE) {
                const int unit = (int)(gb / a.nbands);
                xrow = nullptr;
                if (g < grp.piece_count[unit]) {
                    const int sl = grp.sorted_slot[grp.piece_first[unit] + g];
                    const int xr = a.x_per_slot ? sl : sl / a.topk;
                    xrow = a.x + (size_t)xr * a.K;
                }
            }
        }
        const int left = nb32 - kp * 8;
        chunk_mma<FMT>(codes_ring + (uint32_t)(slot * CB), scales_ring + (uint32_t)(slot * kScaleBytes),
                       xrow, kp * kChunkK, left < 8 ? left : 8, g, t, acc);
    }
    if (i == n) {
        if (cur >= 0)
            flush(cur, acc);
        return;
    }
    // A wait ran out: drain the copies this worker still has in flight
    // (bounded again) so none lands in shared memory after the CTA exits.
    const int issued = (n < i + D) ? n : i + D;
    for (int j = i; j < issued; j++)
        (void)mbar_wait_bounded(bars + 8 * (j % D), (uint32_t)((j / D) & 1));
}

// y[b][n] = sum_s route_w[b][s] * slot_out[b*topk + s][n], in slot order, over
// the slots whose expert index is valid.
__global__ void moe_combine_kernel(const float *slot_out, const int *idx, const float *route_w,
                                   int B, int topk, int N, int E, float *y)
{
    pdl_launch_dependents();
    pdl_wait();
    const int total = B * N;
    for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < total; o += gridDim.x * blockDim.x) {
        const int b = o / N, nn = o - b * N;
        float s = 0.f;
        for (int k = 0; k < topk; k++) {
            const int e = idx[b * topk + k];
            if (e >= 0 && e < E)
                s = fmaf(route_w[b * topk + k], slot_out[(size_t)(b * topk + k) * N + nn], s);
        }
        y[o] = s;
    }
}

// ------------------------------------------------------------------ host ----
namespace {

template <int FMT, bool MOE>
int32_t prepare_kernel()
{
    static bool done[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64 && done[dev])
        return BQ_OK;
    if (cudaFuncSetAttribute((const void *)stream_gemv_kernel<FMT, MOE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes<FMT>()) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64)
        done[dev] = true;
    return BQ_OK;
}

int grid_ctas(long long T)
{
    const int sms = device_sm_count();
    if (sms <= 0)
        return -1;
    long long g = 2LL * sms;
    if (g > kMaxCtas)
        g = kMaxCtas;
    if (T >= 0 && g > T)
        g = T;
    return (int)(g < 1 ? 1 : g);
}

size_t counters_bytes(long long n) { return align_up((size_t)n * sizeof(int), 256); }

template <int FMT>
int32_t gemv_impl(const bq_qmat *W, const uint16_t *x, int32_t B, float *y, void *ws,
                  size_t ws_bytes, int32_t *dev_status, void *stream)
{
    int32_t st = check_qmat(W);
    if (st != BQ_OK)
        return st;
    if (!x || !y || !ws)
        return BQ_ERR_NULL;
    if (B < 1 || B > 8)
        return BQ_ERR_BATCH;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws))
        return BQ_ERR_ALIGN;
    if (ws_bytes < bq_gemv_workspace_bytes(W->N, W->K))
        return BQ_ERR_WORKSPACE;
    st = prepare_kernel<FMT, false>();
    if (st != BQ_OK)
        return st;

    GemvArgs a;
    memset(&a, 0, sizeof(a));
    const int N = W->N, K = W->K;
    const uint64_t cdims[2] = {(uint64_t)(FMT == 4 ? K / 2 : K), (uint64_t)N};
    const uint64_t cstr[1] = {(uint64_t)(FMT == 4 ? K / 2 : K)};
    const uint32_t cbox[2] = {128, (uint32_t)kChunkRows};
    const int ldS = bq_scales_ld(K);
    const uint64_t sdims[2] = {(uint64_t)(K / 32), (uint64_t)N};
    const uint64_t sstr[1] = {(uint64_t)ldS * 2};
    const uint32_t sbox[2] = {8, (uint32_t)kChunkRows};
    if (!encode_tensor_map(&a.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, W->codes, cdims, cstr,
                           cbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&a.tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W->scales, sdims,
                           sstr, sbox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return BQ_ERR_CUDA;
    a.x = reinterpret_cast<const __half *>(x);
    a.out = y;
    a.N = N;
    a.K = K;
    a.B = B;
    a.cpb = (K + kChunkK - 1) / kChunkK;
    a.nbands = (N + kChunkRows - 1) / kChunkRows;
    const long long T = (long long)a.cpb * a.nbands;
    const int G = grid_ctas(T);
    if (G < 0)
        return BQ_ERR_CUDA;
    a.wmax = G * kWarps;
    a.counters = static_cast<int *>(ws);
    a.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + counters_bytes(a.nbands));
    a.status = dev_status;
    void *args[] = {&a};
    cudaError_t e = launch_pdl((const void *)stream_gemv_kernel<FMT, false>, dim3(G), dim3(kThreads),
                               smem_bytes<FMT>(), static_cast<cudaStream_t>(stream), args);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_gemv_workspace_bytes(int32_t N, int32_t K)
{
    if (N < 1 || K < 32 || K % 32 != 0)
        return 0;
    const long long nbands = (N + kChunkRows - 1) / kChunkRows;
    return counters_bytes(nbands) + (size_t)kMaxWorkers * kPartialBytesPerWorker;
}

extern "C" int32_t bq_gemv_q4(const bq_qmat *W, const uint16_t *x, int32_t B, float *y, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return gemv_impl<4>(W, x, B, y, ws, ws_bytes, dev_status, stream);
}

extern "C" int32_t bq_gemv_q8(const bq_qmat *W, const uint16_t *x, int32_t B, float *y, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return gemv_impl<8>(W, x, B, y, ws, ws_bytes, dev_status, stream);
}

extern "C" size_t bq_moe_workspace_bytes(int32_t N, int32_t K, int32_t B, int32_t topk, int32_t E)
{
    if (N < 1 || K < 32 || K % 32 != 0 || B < 1 || B > 8 || topk < 1 || B * topk > kMaxSlots ||
        E < 1 || E > 65535)
        return 0;
    const long long nbands = (N + kChunkRows - 1) / kChunkRows;
    return counters_bytes(nbands * B * topk) + (size_t)kMaxWorkers * kPartialBytesPerWorker +
           align_up((size_t)B * topk * N * sizeof(float), 256);
}

extern "C" int32_t bq_moe_gemv_q4(const bq_qmat *Wstack, int32_t E, int64_t codes_stride,
                                  int64_t scales_stride, const uint16_t *x, int32_t x_per_slot,
                                  const int32_t *expert_idx, const float *route_w, int32_t B,
                                  int32_t topk, float *y, void *ws, size_t ws_bytes,
                                  int32_t *dev_status, void *stream)
{
    int32_t st = check_qmat(Wstack);
    if (st != BQ_OK)
        return st;
    if (!x || !expert_idx || !y || !ws)
        return BQ_ERR_NULL;
    if (B < 1 || B > 8 || B * topk > kMaxSlots)
        return BQ_ERR_BATCH;
    const int N = Wstack->N, K = Wstack->K, ldS = bq_scales_ld(K);
    if (topk < 1 || E < 1 || E > 65535 || codes_stride < (int64_t)N * (K / 2) ||
        scales_stride < (int64_t)N * ldS)
        return BQ_ERR_SHAPE;
    if (codes_stride % 16 != 0 || scales_stride % 8 != 0 || !aligned16(x) || !aligned16(y) ||
        !aligned16(ws) || !aligned16(expert_idx) || (route_w && !aligned16(route_w)))
        return BQ_ERR_ALIGN;
    if (ws_bytes < bq_moe_workspace_bytes(N, K, B, topk, E))
        return BQ_ERR_WORKSPACE;
    st = prepare_kernel<4, true>();
    if (st != BQ_OK)
        return st;

    GemvArgs a;
    memset(&a, 0, sizeof(a));
    const uint64_t cdims[3] = {(uint64_t)(K / 2), (uint64_t)N, (uint64_t)E};
    const uint64_t cstr[2] = {(uint64_t)(K / 2), (uint64_t)codes_stride};
    const uint32_t cbox[3] = {128, (uint32_t)kChunkRows, 1};
    const uint64_t sdims[3] = {(uint64_t)(K / 32), (uint64_t)N, (uint64_t)E};
    const uint64_t sstr[2] = {(uint64_t)ldS * 2, (uint64_t)scales_stride * 2};
    const uint32_t sbox[3] = {8, (uint32_t)kChunkRows, 1};
    if (!encode_tensor_map(&a.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, Wstack->codes, cdims,
                           cstr, cbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&a.tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, Wstack->scales, sdims,
                           sstr, sbox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return BQ_ERR_CUDA;
    const long long nbands = (N + kChunkRows - 1) / kChunkRows;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    float *slot_buf = reinterpret_cast<float *>(wsb + counters_bytes(nbands * B * topk) +
                                                (size_t)kMaxWorkers * kPartialBytesPerWorker);
    a.x = reinterpret_cast<const __half *>(x);
    a.out = route_w ? slot_buf : y;
    a.N = N;
    a.K = K;
    a.B = B;
    a.cpb = (K + kChunkK - 1) / kChunkK;
    a.nbands = (int)nbands;
    const int G = grid_ctas(-1);
    if (G < 0)
        return BQ_ERR_CUDA;
    a.wmax = G * kWarps;
    a.counters = reinterpret_cast<int *>(wsb);
    a.partials = reinterpret_cast<float *>(wsb + counters_bytes(nbands * B * topk));
    a.status = dev_status;
    a.E = E;
    a.topk = topk;
    a.x_per_slot = x_per_slot ? 1 : 0;
    a.idx = expert_idx;
    void *args[] = {&a};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_pdl((const void *)stream_gemv_kernel<4, true>, dim3(G), dim3(kThreads),
                               smem_bytes<4>(), s, args);
    if (e != cudaSuccess)
        return BQ_ERR_CUDA;
    if (route_w) {
        const float *sb = slot_buf;
        int Bv = B, tk = topk, Nv = N, Ev = E;
        void *cargs[] = {(void *)&sb, (void *)&expert_idx, (void *)&route_w, &Bv, &tk, &Nv, &Ev, &y};
        int cg = (B * N + 255) / 256;
        if (cg > 4 * device_sm_count())
            cg = 4 * device_sm_count();
        e = launch_pdl((const void *)moe_combine_kernel, dim3(cg), dim3(256), 0, s, cargs);
        if (e != cudaSuccess)
            return BQ_ERR_CUDA;
    }
    return BQ_OK;
}
