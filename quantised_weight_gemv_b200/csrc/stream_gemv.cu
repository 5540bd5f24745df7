// stream_gemv.cu -- the streamed decode GEMV over block-quantised weights
// (dense Q2-Q6 and Q8, whole decode steps in Q4/Q8, grouped routed-expert
// Q4), sm_100a.
//
// The decode step is a GEMV per quantisation format with the dequantisation
// inside the inner loop (BaseRT, gist.science technical summary,
// "Methodologie" -> "Kernel Fusie en Specialisatie"), and it is bound by
// memory bandwidth ("De 'Big Model' Realiteit"; the follow-up paper's results
// paragraph says the same of its decode path).  The design goal is one thing:
// keep HBM busy with the packed weight bytes and read each of them once.
//
// Work decomposition (stream-K over chunks).  A matrix is cut into bands of
// kRows rows (16 for Q8, Q2, Q3, Q5, Q6; 32 or 16 for Q4, chosen per launch by
// choose_q4_mt) and a band into chunks of 256 weights along K; chunks are
// numbered band-major.  Every warp of the grid is an
// independent worker that owns a ring of shared-memory slots with its own
// mbarriers; its lane 0 keeps TMA loads of the warp's next chunks in flight
// in every slot but the one being read (in a decode step, in every slot: a
// slot is refilled as soon as the warp has read it).  Worker w takes chunks
// [w*cpw, (w+1)*cpw) of a stage, where cpw = ceil(chunks / workers), so every
// SM streams the same number of bytes whatever the matrix shapes.
//
// A band wholly inside one worker's range is written straight to y.  A band
// cut by range boundaries is summed deterministically in two levels: the
// workers of one CTA that touched it combine their fp32 partials (kRows rows x
// 8 columns) in shared memory, the last of them to arrive adding them in
// worker order; if the band continues in other CTAs, that CTA partial goes to
// the workspace with a counted arrival, and the last CTA to arrive adds the
// CTA partials in CTA order, writes y and resets the counter.  No worker waits
// for another.  When the launch runs as thread-block clusters whose
// boundaries are band boundaries (cluster_for), the CTA partials go instead
// straight into the shared memory of the band's first CTA, which waits for
// them and adds them in the same order.
//
// Three modes share that worker loop:
//  - one matrix (bq_gemv_q4 / _q8 / _ex): its descriptor is a kernel
//    parameter; a chain of such launches is a decode step too, each launch
//    loading its first weights while the previous one drains (programmatic
//    dependent launch, BQ_GEMV_STATIC_WEIGHTS);
//  - a decode step (bq_step_run): a plan in device memory lists matrices in
//    stages; stage s+1 may read what stage s wrote (in a model, the next
//    projection's input), so the persistent, co-resident grid passes a grid
//    barrier between stages.  Weight loads never wait for it: a worker's ring
//    runs ahead across stage boundaries, so HBM keeps streaming the next
//    stage's weights while the barrier settles.  The fixed per-token launch
//    and dispatch cost the pages single out for small models (gist.science
//    technical summary, "Resultaten" and "Kernel Fusie") becomes one launch
//    per token;
//  - routed experts (bq_moe_gemv_q4 / _ex): every CTA sorts the (token, slot) ->
//    expert list (at most 64 entries) in shared memory, which gives the same
//    grouping on every CTA without a separate kernel; each distinct expert,
//    cut into pieces of at most 8 routed slots (the mma's N), becomes one
//    matrix of the numbering, so each routed expert's weights are read once
//    for all of its tokens.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {

constexpr int kMaxSlots = 64;   // B * topk
constexpr int kModeMatrix = 0, kModePlan = 1, kModeMoE = 2;
constexpr uint32_t kPlanMagic = 0x42515031u;   // "BQP1"

struct alignas(64) MatDesc {
    CUtensorMap tm_codes;
    CUtensorMap tm_scales;
    const __half *x;     // [B][K]
    float *y;            // [B][N]
    int N, K, B;
    int cpb;             // chunks per band
    int nbands;
    int chunk_base;      // first chunk of this matrix within its stage
    int band_base;       // first arrival counter of this matrix within its stage
    int epi;             // BQ_EPI_*
};

// The per-matrix fields the worker loop reads (everything but the tensor
// maps), cached in shared memory so cursor moves, band changes and flushes
// never wait on global memory.
struct MatInfo {
    const __half *x;
    float *y;
    int N, K, B, cpb, nbands, chunk_base, band_base, epi;
};

constexpr int kMaxPlanMats = 256;   // plan size limit (shared-memory cache)

struct StageDesc {
    int mat_begin, mat_end;
    int T;               // chunks in the stage
    int cpw;             // chunks per worker
    int W;               // workers with a non-empty range
    int nbands;          // bands in the stage
};

struct PlanHeader {
    uint32_t magic;
    int fmt, n_mats, n_stages, grid, max_stage_bands;
    uint64_t stages_off, mats_off;   // byte offsets from the plan base
};

struct KernelArgs {
    MatDesc mat0;                    // matrix / routed-expert modes
    StageDesc stage0;
    const MatDesc *mats;             // plan mode (device memory)
    const StageDesc *stages;
    int n_stages;
    int n_mats;
    int wmax;                        // gridDim.x * kWarps
    int *counters;                   // per band of a stage; zero on entry and exit
    float *partials;                 // [CTA][slot 0/1][kMT][32 lanes] float4 (cross-CTA band sums)
    int *status;                     // device status word or null
    int prefill;                     // matrix mode: load weights before the PDL wait
    unsigned *sync;                  // plan mode: [0] arrivals, [64] exits (separate lines)
    long long wait_cycles;           // plan mode: limit of a grid-barrier wait (SM cycles)
    int extra_arrivals;              // plan mode: arrivals a barrier waits for beyond the grid's
    // routed experts
    int E, topk, x_per_slot;
    const int *idx;
    // Q3 / Q5 / Q6 (matrix mode): the top-bit plane of mat0's codes
    alignas(64) CUtensorMap tm_codes_hi;
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
__device__ void group_experts(const KernelArgs &a, ExpertGroups &grp)
{
    const int lane = threadIdx.x & 31;
    const int M = a.mat0.B * a.topk;
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

// Position of a chunk inside a stage: matrix (or expert piece) u, band, k-piece,
// with the current unit's geometry cached in registers.
struct Cursor {
    int s;        // stage
    int u;        // matrix index (plan: global; otherwise 0 / piece)
    int band, kp;
    int c, c_end; // chunk index within the stage and end of this worker's range
    int cpb, nbands;
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <int FMT, int MODE, int MTQ = default_mt<FMT>(), bool CL = false>
__global__ void __launch_bounds__(kThreads, BQ_MIN_BLOCKS) stream_gemv_kernel(const __grid_constant__ KernelArgs a)
{
    using F = Fmt<FMT, MTQ>;
    constexpr int D = F::kStages;
    constexpr int CB = F::kCodeBytes;
    constexpr int SB = F::kScaleBytes;
    constexpr int MT = F::kMT;
    constexpr int ROWS = F::kRows;
    constexpr uint32_t kTx = F::kCodeLoad + SB;   // bytes one chunk's loads bring
    constexpr bool MOE = MODE == kModeMoE;
    constexpr bool PLAN = MODE == kModePlan;

    extern __shared__ uint8_t smem_raw[];
    __shared__ ExpertGroups grp;
    __shared__ int cta_arrivals;
    __shared__ int local_ctr[kWarps];   // arrivals of CTA-local split bands
    __shared__ alignas(8) uint64_t stage_bar;
    __shared__ int stage_failed;        // PLAN: a grid-barrier wait ran out
    __shared__ alignas(8) uint64_t cl_bar;   // CL: cross-CTA partials received

    uint8_t *sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    uint8_t *codes_ring = sbase + warp * D * CB;
    uint8_t *scales_ring = sbase + kWarps * D * CB + warp * D * SB;
    const uint32_t bars = smem_u32(sbase + kWarps * D * (CB + SB) + warp * D * 8);
    // Per-warp partial sums of CTA-local split bands: [warp][slot][mt][lane].
    float4 *local_part = reinterpret_cast<float4 *>(sbase + kWarps * D * (CB + SB) + kWarps * D * 8);
    // Descriptor cache: stage table then matrix info (one entry each outside
    // plan mode).
    StageDesc *stg = reinterpret_cast<StageDesc *>(local_part + kWarps * 2 * MT * 32);
    const int n_stages = PLAN ? a.n_stages : 1;
    MatInfo *minfo = reinterpret_cast<MatInfo *>(stg + n_stages);
    // CL (matrix mode, launched as clusters whose boundaries are band
    // boundaries): the partials other CTAs of the cluster send for the band
    // this CTA finishes, [sender - this CTA - 1][mt][lane] float4, after the
    // descriptor cache (one matrix).
    static_assert(!CL || MODE == kModeMatrix, "cluster sums are a matrix-mode path");
    const uint32_t cl_recv = CL ? (smem_u32(minfo + 1) + 15u) / 16u * 16u : 0u;
    const MatDesc *mats = PLAN ? a.mats : &a.mat0;   // tensor maps stay in global / param space
    {
        const int n_m = PLAN ? a.n_mats : 1;
        for (int i = threadIdx.x; i < n_stages; i += kThreads)
            stg[i] = PLAN ? a.stages[i] : a.stage0;
        for (int i = threadIdx.x; i < n_m; i += kThreads) {
            const MatDesc &m = mats[i];
            MatInfo mi;
            mi.x = m.x;
            mi.y = m.y;
            mi.N = m.N;
            mi.K = m.K;
            mi.B = m.B;
            mi.cpb = m.cpb;
            mi.nbands = m.nbands;
            mi.chunk_base = m.chunk_base;
            mi.band_base = m.band_base;
            mi.epi = m.epi;
            minfo[i] = mi;
        }
    }

    if (lane == 0) {
        for (int s = 0; s < D; s++)
            mbar_init(bars + 8 * s, 1);
    }
    if (threadIdx.x < kWarps)
        local_ctr[threadIdx.x] = 0;
    if (PLAN && threadIdx.x == 0) {
        cta_arrivals = 0;
        stage_failed = 0;
        mbar_init(smem_u32(&stage_bar), 1);
    }
    if (CL && threadIdx.x == 0) {
        mbar_init(smem_u32(&cl_bar), 1);
        fence_mbarrier_init_cluster();
    }
    if (lane == 0)
        fence_barrier_init();

    pdl_launch_dependents();
    // Everything below reads inputs or writes outputs and the workspace, so it
    // waits for the previous kernel on the stream to complete -- except, when
    // the caller declared the weights static, the first weight loads of the
    // ring (matrix mode), issued before the wait further down.
    const bool prefill = !MOE && !PLAN && a.prefill;
    if (!prefill)
        pdl_wait();

    if constexpr (MOE) {
        if (warp == 0)
            group_experts(a, grp);
        __syncthreads();
        // CTA 0 reports invalid indices and zeroes their per-slot outputs.
        if (blockIdx.x == 0 && grp.nvalid < a.mat0.B * a.topk) {
            if (threadIdx.x == 0 && a.status)
                atomicOr(a.status, kStatusExpertIndex);
            for (int i = 0; i < a.mat0.B * a.topk; i++) {
                if (grp.key[i] != 0x7fffffff)
                    continue;
                if (a.mat0.epi == BQ_EPI_SWIGLU) {
                    __half *h = reinterpret_cast<__half *>(a.mat0.y);
                    const int F = a.mat0.N / 2;
                    for (int r = threadIdx.x; r < F; r += kThreads)
                        h[(size_t)i * F + r] = __float2half_rn(0.0f);
                } else {
                    for (int r = threadIdx.x; r < a.mat0.N; r += kThreads)
                        a.mat0.y[(size_t)i * a.mat0.N + r] = 0.f;
                }
            }
        }
        if (threadIdx.x == 0) {
            StageDesc st = a.stage0;
            st.nbands = grp.npieces * a.mat0.nbands;
            st.T = st.nbands * a.mat0.cpb;
            st.cpw = (st.T + a.wmax - 1) / a.wmax;
            if (st.cpw < 1)
                st.cpw = 1;
            st.W = (st.T + st.cpw - 1) / st.cpw;
            stg[0] = st;
        }
        __syncthreads();
    } else {
        __syncthreads();
        // Every CTA's receive barrier is initialised before any CTA of the
        // cluster can send to it.
        if constexpr (CL)
            cluster_sync_all();
    }

    // Workers are numbered CTA-major, so a band split among consecutive
    // workers usually lies within one CTA and is summed in shared memory.
    const int w = blockIdx.x * kWarps + warp;
    const int cta_first = blockIdx.x * kWarps;
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_s = policy_evict_normal();

    // Per-unit geometry (matrix, or expert piece in MoE mode).  Only plan mode
    // indexes a descriptor array; the other modes have one descriptor.
    auto unit_mat = [&](int u) -> const MatInfo & { return minfo[PLAN ? u : 0]; };
    auto unit_cpb = [&](int u) { return unit_mat(u).cpb; };
    auto unit_chunk_base = [&](int u) {
        return PLAN ? minfo[u].chunk_base : (MOE ? u * a.mat0.nbands * a.mat0.cpb : 0);
    };
    auto unit_band_base = [&](int u) {
        return PLAN ? minfo[u].band_base : (MOE ? u * a.mat0.nbands : 0);
    };

    // Place a cursor at the first chunk of this worker's range in stage s, or
    // at the first later stage where the range is non-empty.  Returns false
    // when no stage >= s has work for this worker.
    auto seek = [&](Cursor &cu, int s) -> bool {
        for (; s < n_stages; s++) {
            const StageDesc &st = stg[s];
            if (w >= st.W)
                continue;
            const int c0 = w * st.cpw;
            const int c1 = min(c0 + st.cpw, st.T);
            int u = MOE ? c0 / (a.mat0.nbands * a.mat0.cpb) : (PLAN ? st.mat_begin : 0);
            if (PLAN)
                while (u + 1 < st.mat_end && minfo[u + 1].chunk_base <= c0)
                    u++;
            const int rel = c0 - unit_chunk_base(u);
            cu.s = s;
            cu.u = u;
            cu.cpb = unit_mat(u).cpb;
            cu.nbands = unit_mat(u).nbands;
            cu.band = rel / cu.cpb;
            cu.kp = rel - cu.band * cu.cpb;
            cu.c = c0;
            cu.c_end = c1;
            return true;
        }
        cu.s = n_stages;
        return false;
    };
    auto advance = [&](Cursor &cu) {
        cu.c++;
        if (cu.c == cu.c_end) {
            seek(cu, cu.s + 1);
            return;
        }
        if (++cu.kp == cu.cpb) {
            cu.kp = 0;
            if (++cu.band == cu.nbands) {
                cu.band = 0;
                cu.u++;
                if (PLAN) {
                    cu.cpb = minfo[cu.u].cpb;
                    cu.nbands = minfo[cu.u].nbands;
                }
            }
        }
    };

    // Chunks left in the cursor's current run: consecutive chunks of one
    // band inside the worker's range.
    auto run_left = [&](const Cursor &cu) { return min(cu.cpb - cu.kp, cu.c_end - cu.c); };

    Cursor iss;
    bool iss_live = seek(iss, 0);
    int iss_left = iss_live ? run_left(iss) : 0;
    int issued = 0;
    // Plan mode: the TMA unit must fetch a matrix's tensor maps from global
    // memory before its first load; prefetch them one load ahead of the issue
    // cursor so no load waits for a descriptor.
    int prefetched_u = -1;
    auto prefetch_maps = [&](int u) {
        if constexpr (PLAN) {
            if (lane == 0 && u > prefetched_u && u < a.n_mats) {
                prefetch_tensormap(&mats[u].tm_codes);
                prefetch_tensormap(&mats[u].tm_scales);
                prefetched_u = u;
            }
        }
    };
    if (iss_live) {
        prefetch_maps(iss.u);
        prefetch_maps(iss.u + 1);
    }
    auto issue_one = [&]() {
        if (lane == 0) {
            const int slot = issued % D;
            const uint32_t bar = bars + 8 * slot;
            const uint32_t cdst = smem_u32(codes_ring + slot * CB);
            const uint32_t sdst = smem_u32(scales_ring + slot * SB);
            const int row = iss.band * ROWS;
            mbar_arrive_expect_tx(bar, kTx);
            if constexpr (MOE) {
                const int e = grp.piece_expert[iss.u];
                tma_load_3d(cdst, &a.mat0.tm_codes, bar, iss.kp * 128, row, e, pol);
                tma_load_3d(sdst, &a.mat0.tm_scales, bar, iss.kp * 8, row, e, (FMT == 4) ? pol : pol_s);
            } else {
                const MatDesc &m = mats[PLAN ? iss.u : 0];
#pragma unroll
                for (int bx = 0; bx < F::kBoxes; bx++)
                    tma_load_2d(cdst + bx * (ROWS * F::kLoRow), &m.tm_codes, bar,
                                iss.kp * F::kLoRow * F::kBoxes + bx * F::kLoRow, row, pol);
                if constexpr (FMT == 3 || FMT == 5 || FMT == 6)
                    tma_load_2d(cdst + ROWS * F::kLoRow, &a.tm_codes_hi, bar, iss.kp * F::kTopRow,
                                row, pol);
                tma_load_2d(sdst, &m.tm_scales, bar, iss.kp * 8, row, (FMT == 4) ? pol : pol_s);
            }
        }
        issued++;
        if (--iss_left > 0) {   // next chunk of the same run
            iss.kp++;
            iss.c++;
            return;
        }
        advance(iss);
        iss_live = iss.s < n_stages;
        if (iss_live) {
            iss_left = run_left(iss);
            prefetch_maps(iss.u);   // the matrix of the next load this warp issues
        }
    };

    // Fill the ring.  Plan mode keeps every slot loading (see the refill
    // below); the other modes run one slot behind, refilling a slot at the
    // top of the next chunk, after that chunk's x loads are in flight -- but
    // fill every slot when the loads run ahead of the wait for the previous
    // kernel.
    while (iss_live && issued < ((PLAN || prefill) ? D : D - 1))
        issue_one();

    bool ok = true;
    int sw[8];
    lane_swizzle<FMT>(g, sw);
    // 16 in a register the compiler cannot see through, so the Q4 nibble
    // placement multiplies on the FMA pipe instead of shifting on the ALU.
    const uint32_t m16 = launder(16u);
    if (prefill)
        pdl_wait();

    // Output of one band: acc[mt] holds (row 16mt+g, col 2t), (row 16mt+g,
    // col 2t+1), (row 16mt+g+8, col 2t), (row 16mt+g+8, col 2t+1).
    auto store_band = [&](int u, int band, const float (&v)[MT][4]) {
        // The descriptor fields and this lane's two output columns are read
        // into registers first: the output pointer is a generic one, so
        // otherwise every store would force shared-memory reloads.
        const MatInfo &mref = unit_mat(u);
        const int N = mref.N, epi = mref.epi;
        float *const y = mref.y;
        int out[2];                      // output row of batch column (or piece slot) 2t + c; -1: none
#pragma unroll
        for (int c = 0; c < 2; c++) {
            const int col = 2 * t + c;
            if constexpr (MOE)
                out[c] = col < grp.piece_count[u] ? grp.sorted_slot[grp.piece_first[u] + col] : -1;
            else
                out[c] = col < mref.B ? col : -1;
        }
        if (epi == BQ_EPI_SWIGLU) {
            // SwiGLU pair order: in each 16-row tile, rows 0-7 are gate rows
            // and rows 8-15 the up rows of the same 8 outputs, so this lane
            // holds gate (v[mt][c]) and up (v[mt][2 + c]) of output i for
            // batch column (or expert-piece slot) 2t + c.  h = silu(g) * u in
            // fp32, stored as fp16.
            __half *const h = reinterpret_cast<__half *>(y);
            const int F = N / 2;
#pragma unroll
            for (int mt = 0; mt < MT; mt++) {
                const int i = (band * ROWS + 16 * mt) / 2 + g;
                if (i >= F)
                    continue;
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    if (out[c] < 0)
                        continue;
                    const float gv = v[mt][c] * unscale<FMT>();
                    const float uv = v[mt][2 + c] * unscale<FMT>();
                    // silu(g) * u with the fast exp and divide (a few fp32
                    // ulp, far below the fp16 rounding that follows); for g
                    // below about -88 the divisor is inf and the result 0.
                    h[(size_t)out[c] * F + i] = __float2half_rn(__fdividef(gv, 1.0f + __expf(-gv)) * uv);
                }
            }
            return;
        }
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int row = band * ROWS + 16 * mt + g + ((q & 2) ? 8 : 0);
                const int o = out[q & 1];
                if (row < N && o >= 0)
                    y[(size_t)o * N + row] = v[mt][q] * unscale<FMT>();
            }
        }
    };

    // Cross-CTA partials: [CTA][slot 0/1][mt][lane] float4.  A CTA has at
    // most two bands that continue into other CTAs in a stage: the one holding
    // its first chunk (slot 0) and the one holding its last (slot 1).
    auto part_at = [&](int c, int sl, int mt) {
        return reinterpret_cast<float4 *>(a.partials) + (((size_t)c * 2 + sl) * MT + mt) * 32 + lane;
    };
    // Writes the band's finished sum to y when this worker is the last to
    // contribute; `acc` (this worker's partial) is used as scratch.
    auto flush = [&](int s, int u, int band, float (&acc)[MT][4]) {
        const StageDesc &st = stg[s];
        const int cpw = st.cpw;
        const int cpb = unit_cpb(u);
        const int bs = unit_chunk_base(u) + band * cpb, be = bs + cpb;
        const int c0 = w * cpw, c1 = min(c0 + cpw, st.T);
        if (bs >= c0 && be <= c1) {
            store_band(u, band, acc);
            return;
        }
        // Workers wf..wl share the band; lf..ll of them are warps of this CTA.
        const int wf = bs / cpw, wl = (be - 1) / cpw;
        const int lf = max(wf, cta_first), ll = min(wl, cta_first + kWarps - 1);
        if (ll > lf) {
            // Level 1, in shared memory: each of the CTA's workers stores its
            // partial and bumps the band's CTA counter (slot lf - cta_first,
            // unique among the CTA's open bands) with CTA-scope release; the
            // last to arrive acquires and adds the partials in worker order.
            // Nobody waits.
            const int myslot = (c0 >= bs) ? 0 : 1;
#pragma unroll
            for (int mt = 0; mt < MT; mt++)
                local_part[((warp * 2 + myslot) * MT + mt) * 32 + lane] =
                    make_float4(acc[mt][0], acc[mt][1], acc[mt][2], acc[mt][3]);
            __syncwarp();
            int lold = 0;
            if (lane == 0)
                asm volatile("atom.acq_rel.cta.shared::cta.add.s32 %0, [%1], 1;"
                             : "=r"(lold) : "r"(smem_u32(&local_ctr[lf - cta_first])) : "memory");
            lold = __shfl_sync(0xffffffffu, lold, 0);
            if (lold != ll - lf)
                return;
            __syncwarp();
#pragma unroll
            for (int mt = 0; mt < MT; mt++)
                acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
            for (int v = lf; v <= ll; v++) {
                const int sl = (v * cpw >= bs) ? 0 : 1;
#pragma unroll
                for (int mt = 0; mt < MT; mt++) {
                    const float4 p = local_part[(((v - cta_first) * 2 + sl) * MT + mt) * 32 + lane];
                    acc[mt][0] += p.x;
                    acc[mt][1] += p.y;
                    acc[mt][2] += p.z;
                    acc[mt][3] += p.w;
                }
            }
            if (lane == 0)
                local_ctr[lf - cta_first] = 0;
        }
        if (wf >= cta_first && wl < cta_first + kWarps) {
            store_band(u, band, acc);
            return;
        }
        const int cf = wf / kWarps, cl = wl / kWarps;
        if constexpr (CL) {
            // Level 2 inside the cluster (the host launches clusters only when
            // no band crosses one): the band's other CTAs store their partial
            // straight into the shared memory of its first CTA, which waits
            // for them, adds all in CTA order and stores y.  Each CTA finishes
            // at most one such band (its last one) and sends for at most one
            // (its first one), so one receive area and one mbarrier phase per
            // launch suffice.
            const uint32_t C = cluster_nctarank();
            const uint32_t first_rank = (uint32_t)cf % C;
            if (blockIdx.x != (unsigned)cf) {
                const uint32_t slot = cl_recv + ((uint32_t)(blockIdx.x - cf - 1) * MT * 32 + lane) * 16;
                const uint32_t rbar = mapa_shared(smem_u32(&cl_bar), first_rank);
#pragma unroll
                for (int mt = 0; mt < MT; mt++)
                    st_async_v4(mapa_shared(slot + mt * 512, first_rank),
                                make_float4(acc[mt][0], acc[mt][1], acc[mt][2], acc[mt][3]), rbar);
                return;
            }
            if (lane == 0)
                mbar_arrive_expect_tx(smem_u32(&cl_bar), (uint32_t)((cl - cf) * MT * 512));
            if (!__all_sync(0xffffffffu, mbar_wait_cluster_bounded(smem_u32(&cl_bar), 0u))) {
                if (lane == 0 && a.status)
                    atomicOr(a.status, kStatusTimeout);
                return;
            }
            float sum[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; mt++) {
                sum[mt][0] = 0.f + acc[mt][0];
                sum[mt][1] = 0.f + acc[mt][1];
                sum[mt][2] = 0.f + acc[mt][2];
                sum[mt][3] = 0.f + acc[mt][3];
            }
            for (int v = cf + 1; v <= cl; v++) {
#pragma unroll
                for (int mt = 0; mt < MT; mt++) {
                    const float4 p = lds128_f32(cl_recv + (((uint32_t)(v - cf - 1) * MT + mt) * 32 + lane) * 16);
                    sum[mt][0] += p.x;
                    sum[mt][1] += p.y;
                    sum[mt][2] += p.z;
                    sum[mt][3] += p.w;
                }
            }
            store_band(u, band, sum);
            return;
        }
        // Level 2, the band continues in other CTAs: one partial per CTA
        // through the workspace and a counted arrival; the last CTA to arrive
        // adds the partials in CTA order, stores y and resets the counter.
        const int cslot = (bs <= cta_first * cpw) ? 0 : 1;
#pragma unroll
        for (int mt = 0; mt < MT; mt++)
            __stcg(part_at(blockIdx.x, cslot, mt), make_float4(acc[mt][0], acc[mt][1], acc[mt][2], acc[mt][3]));
        // The warp's partial stores happen before lane 0's release increment
        // (__syncwarp orders them); the last arriver's acquire increment then
        // makes every partial visible to the whole warp (__syncwarp again).
        __syncwarp();
        int *ctr = a.counters + unit_band_base(u) + band;
        int old = 0;
        if (lane == 0)
            old = atom_add_acq_rel_gpu(ctr, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != cl - cf)
            return;
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < MT; mt++)
            acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        // Two CTAs' partials in flight at a time.  Each slot is cleared once
        // read, so the workspace is all-zero again when the launch ends and
        // any later call, of any shape, can use it.
        const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int v = cf; v <= cl; v += 2) {
            const int v1 = min(v + 1, cl);
            const int sl0 = (bs <= v * kWarps * cpw) ? 0 : 1;
            const int sl1 = (bs <= v1 * kWarps * cpw) ? 0 : 1;
            float4 p0[MT], p1[MT];
#pragma unroll
            for (int mt = 0; mt < MT; mt++) {
                p0[mt] = __ldcg(part_at(v, sl0, mt));
                p1[mt] = __ldcg(part_at(v1, sl1, mt));
            }
#pragma unroll
            for (int mt = 0; mt < MT; mt++) {
                __stcg(part_at(v, sl0, mt), zero4);
                __stcg(part_at(v1, sl1, mt), zero4);
            }
#pragma unroll
            for (int mt = 0; mt < MT; mt++) {
                acc[mt][0] += p0[mt].x;
                acc[mt][1] += p0[mt].y;
                acc[mt][2] += p0[mt].z;
                acc[mt][3] += p0[mt].w;
            }
            if (v1 > v) {
#pragma unroll
                for (int mt = 0; mt < MT; mt++) {
                    acc[mt][0] += p1[mt].x;
                    acc[mt][1] += p1[mt].y;
                    acc[mt][2] += p1[mt].z;
                    acc[mt][3] += p1[mt].w;
                }
            }
        }
        store_band(u, band, acc);
        if (lane == 0)
            *ctr = 0;
    };

    // Grid barrier between stages (plan mode; the launch is cooperative, so
    // every CTA is resident).  Each warp's lane 0 arrives on a CTA counter
    // with CTA-scope release; the CTA's last warp acquires it, adds one
    // GPU-scope release arrival to the grid counter (a fire-and-forget
    // reduction; release is cumulative, so it publishes every warp's y
    // stores) and polls the counter (acquire, short back-off) until all CTAs
    // have arrived, then releases its CTA's warps through a shared mbarrier.
    // Every wait is bounded: the grid poll by a.wait_cycles, after which it
    // reports BQ_ERR_TIMEOUT, marks the CTA's barrier failed and still
    // releases the CTA's warps, which then stop (drain their copies, exit).
    // a.extra_arrivals > 0 asks for arrivals no CTA makes: the way a test
    // makes the expiry path run without a fault or a missing CTA.
    auto stage_arrive_and_wait = [&](int s) {
        __syncwarp();
        if (lane == 0) {
            int old;
            asm volatile("atom.acq_rel.cta.shared::cta.add.s32 %0, [%1], 1;"
                         : "=r"(old) : "r"(smem_u32(&cta_arrivals)) : "memory");
            if (old == kWarps * (s + 1) - 1) {
                const unsigned target = (gridDim.x + (unsigned)a.extra_arrivals) * (unsigned)(s + 1);
                asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&a.sync[0]) : "memory");
                const long long t0 = clock64();
                while (ld_acquire_gpu(&a.sync[0]) < target) {
                    if (clock64() - t0 > a.wait_cycles) {
                        if (a.status)
                            atomicOr(a.status, kStatusTimeout);
                        stage_failed = 1;
                        break;
                    }
                    __nanosleep(32);
                }
                // (the mbarrier arrive releases the stage_failed store to
                // the CTA's warps, whose wait acquires it)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&stage_bar))
                             : "memory");
            }
        }
        __syncwarp();
        if (!mbar_wait_bounded(smem_u32(&stage_bar), (uint32_t)(s & 1))) {
            if (lane == 0 && a.status)
                atomicOr(a.status, kStatusTimeout);
            ok = false;
        }
        if (*(volatile int *)&stage_failed)
            ok = false;
    };

    Cursor cur;
    bool live = seek(cur, 0);
    int done = 0;                  // chunks consumed (ring index)
    float acc[MT][4];
    int acc_u = -1, acc_band = -1; // band the accumulators belong to
    const __half *xrow = nullptr;
    int pf_blocks = 0;             // x prefetch: next chunk's blocks, 0 when the rows would crowd L1
    int nb32 = 0;

    for (int s = 0; s < n_stages; s++) {
        if (s > 0) {
            stage_arrive_and_wait(s - 1);
            if (!ok)
                break;
        }
        while (live && cur.s == s) {
            if (cur.u != acc_u || cur.band != acc_band) {
                if (acc_u >= 0)
                    flush(s, acc_u, acc_band, acc);
#pragma unroll
                for (int mt = 0; mt < MT; mt++)
                    acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
                if (cur.u != acc_u) {
                    const MatInfo &m = unit_mat(cur.u);
                    nb32 = m.K / kBlock;
                    if constexpr (MOE) {
                        const int col = min(g, grp.piece_count[cur.u] - 1);
                        const int sl = grp.sorted_slot[grp.piece_first[cur.u] + col];
                        xrow = m.x + (size_t)(a.x_per_slot ? sl : sl / a.topk) * m.K;
                    } else {
                        xrow = m.x + (size_t)min(g, m.B - 1) * m.K;
                        pf_blocks = m.B <= 2 ? 8 : 0;
                    }
                }
                acc_u = cur.u;
                acc_band = cur.band;
            }
            // One chunk of the run: x first (its latency then overlaps the
            // TMA issue and the wait), then (outside plan mode) the load of a
            // later chunk into the slot freed last round, then this chunk's
            // weights.  Called with a literal nblk of 8 for full chunks, so
            // their code has no per-block bounds.
            auto one_chunk = [&](const __half *xp, int nblk, int next_nblk) -> bool {
                uint2 xa[8], xb[8];
                chunk_load_x<PLAN>(xp, nblk, xa, xb);
                // The run's next chunk (next_nblk blocks, 0: none): pull its
                // x into L1 now, so its loads do not wait a full L2 round
                // trip after this chunk's compute.  Lane t fetches the
                // 128-byte line t of its row's 512 bytes.  Only for B <= 2:
                // L1 is what shared memory leaves (~28 KB an SM), and 16
                // warps' next chunks at B = 8 (64 KB) measured slower.
                if (2 * t < min(next_nblk, pf_blocks))
                    prefetch_l1(xp + kChunkK + 60 * t);
                if (!PLAN && iss_live && issued < done + D) {
                    __syncwarp();
                    issue_one();
                }
                const int slot = done % D;
                if (!mbar_wait_bounded(bars + 8 * slot, (uint32_t)((done / D) & 1))) {
                    if (lane == 0 && a.status)
                        atomicOr(a.status, kStatusTimeout);
                    return false;
                }
                // Shared addresses of the slot, ordered after its wait (launder).
                const uint32_t cs = launder(smem_u32(codes_ring + slot * CB));
                const uint32_t ss = launder(smem_u32(scales_ring + slot * SB));
                chunk_mma<FMT, MT>(cs, ss, nblk, g, t, sw, xa, xb, acc, m16);
                done++;
                // Plan mode: refill the slot just read at once, before any
                // flush or stage barrier, so the ring always holds the warp's
                // next D chunks -- across stage boundaries too.  (The
                // __syncwarp orders every lane's reads of the slot before lane
                // 0 issues the copy.)
                if (PLAN && iss_live) {
                    __syncwarp();
                    issue_one();
                }
                return true;
            };
            // The run: consecutive chunks of this band inside the worker's
            // range; only the band's last chunk can be partial (K not a
            // multiple of 256).
            const int run = run_left(cur);
            const int tail = nb32 - (cur.cpb - 1) * 8;   // blocks in the band's last chunk
            const int nfull = (cur.kp + run == cur.cpb && tail < 8) ? run - 1 : run;
            const __half *xp = xrow + cur.kp * kChunkK + 4 * t;
            for (int i = 0; i < nfull && ok; i++, xp += kChunkK)
                ok = one_chunk(xp, 8, i + 1 < nfull ? 8 : (nfull < run ? tail : 0));
            if (ok && nfull < run)
                ok = one_chunk(xp, tail, 0);
            if (!ok)
                break;
            // Step the cursor past the run (its last step may change band,
            // matrix or stage).
            cur.c += run - 1;
            cur.kp += run - 1;
            advance(cur);
            live = cur.s < n_stages;
        }
        if (!ok)
            break;
        if (acc_u >= 0) {
            flush(s, acc_u, acc_band, acc);
            acc_u = acc_band = -1;
        }
    }

    if (!ok) {
        // A wait ran out: drain the copies this worker still has in flight
        // (bounded again) so none lands in shared memory after the CTA exits.
        for (int j = done; j < issued; j++)
            (void)mbar_wait_bounded(bars + 8 * (j % D), (uint32_t)((j / D) & 1));
    }
    if constexpr (PLAN) {
        // The last CTA to leave resets the barrier counters for the next launch.
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            const unsigned old = atomicAdd(&a.sync[64], 1u);
            if (old == gridDim.x - 1) {
                a.sync[0] = 0;
                a.sync[64] = 0;
                __threadfence();
            }
        }
    }
}

// y[b][n] = sum_s route_w[b][s] * slot_out[b*topk + s][n], in slot order, over
// the slots whose expert index is valid.
// Each slot value is cleared once read, leaving the workspace all-zero.
__global__ void moe_combine_kernel(float *slot_out, const int *idx, const float *route_w,
                                   int B, int topk, int N, int E, float *y)
{
    pdl_launch_dependents();
    pdl_wait();
    const int total = B * N;
    for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < total; o += gridDim.x * blockDim.x) {
        const int b = o / N, nn = o - b * N;
        float s = 0.f;
        // eight slots' loads in flight, then their stores of zero
        for (int k0 = 0; k0 < topk; k0 += 8) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int k = k0 + j;
                const int e = k < topk ? idx[b * topk + k] : -1;
                v[j] = (e >= 0 && e < E) ? slot_out[(size_t)(b * topk + k) * N + nn] : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int k = k0 + j;
                if (k < topk) {
                    const int e = idx[b * topk + k];
                    if (e >= 0 && e < E) {
                        s = fmaf(route_w[b * topk + k], v[j], s);
                        slot_out[(size_t)(b * topk + k) * N + nn] = 0.f;
                    }
                }
            }
        }
        y[o] = s;
    }
}

// ------------------------------------------------------------------ host ----
namespace {

// Dynamic shared memory of a launch: the rings plus the descriptor cache.
template <int FMT, int MT = default_mt<FMT>()>
constexpr size_t launch_smem(int n_stages, int n_mats, bool cl = false)
{
    return (size_t)smem_bytes<FMT, MT>() + (size_t)kWarps * 2 * MT * 32 * sizeof(float4) +
           (size_t)n_stages * sizeof(StageDesc) + (size_t)n_mats * sizeof(MatInfo) +
           (cl ? 16 + (size_t)(kMaxCluster - 1) * MT * 32 * sizeof(float4) : 0);
}

template <int FMT, int MODE, int MT = default_mt<FMT>(), bool CL = false>
int32_t prepare_kernel()
{
    // Per device: the attribute is set once.  Atomic, since host threads may
    // launch concurrently (two of them setting it twice is harmless).
    static std::atomic<bool> done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire))
        return BQ_OK;
    if (cudaFuncSetAttribute((const void *)stream_gemv_kernel<FMT, MODE, MT, CL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)launch_smem<FMT, MT>(MODE == kModePlan ? kMaxPlanMats : 1,
                                                       MODE == kModePlan ? kMaxPlanMats : 1, CL)) !=
        cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64)
        done[dev].store(true, std::memory_order_release);
    return BQ_OK;
}

// CTAs of one launch: BQ_MIN_BLOCKS per SM (the kernel's occupancy), capped.
int max_ctas()
{
    const int sms = device_sm_count();
    if (sms <= 0)
        return -1;
    return std::min(BQ_MIN_BLOCKS * sms, kMaxCtas);
}

size_t counters_bytes(long long n) { return align_up((size_t)n * sizeof(int), 256); }
constexpr size_t kPartialsBytes = (size_t)kMaxCtas * kPartialBytesPerCta;
constexpr size_t kSyncBytes = 512;

// L2 fill widths: a code box row is 128 bytes (promote to exactly that); a
// scale box row is 16 bytes of a longer row, and a wider fill would pull in
// bytes of the neighbouring row too (measured: ~7% extra DRAM reads at 256 B).
constexpr CUtensorMapL2promotion kPromoCodes = CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
constexpr CUtensorMapL2promotion kPromoScales = CU_TENSOR_MAP_L2_PROMOTION_NONE;

int rows_of(int fmt) { return fmt == 4 ? Fmt<4>::kRows : Fmt<8>::kRows; }   // (Q2-Q6: 16 as Q8)

// R: rows per chunk (the band height), rows_of(fmt) unless a launch chose
// another Q4 geometry.
bool fill_matdesc(int fmt, const bq_qmat *W, const uint16_t *x, int B, float *y, MatDesc *m,
                  int R = 0)
{
    if (R == 0)
        R = rows_of(fmt);
    const int N = W->N, K = W->K;
    // The first plane of each row: Q5 / Q6 the low-nibble plane, the first
    // K/2 bytes of each 5K/8- or 3K/4-byte row; Q3 the 2-bit plane, the first
    // K/4 bytes of each 3K/8-byte row (Q2: all of a K/4-byte row), in 64-byte
    // boxes under the 64-byte swizzle.
    const bool low2 = fmt == 2 || fmt == 3;
    const uint64_t cdims[2] = {(uint64_t)(fmt == 8 ? K : low2 ? K / 4 : K / 2), (uint64_t)N};
    const uint64_t cstr[1] = {(uint64_t)(fmt == 2   ? K / 4
                                         : fmt == 3 ? 3 * K / 8
                                         : fmt == 4 ? K / 2
                                         : fmt == 5 ? 5 * K / 8
                                         : fmt == 6 ? 3 * K / 4 : K)};
    const uint32_t cbox[2] = {low2 ? 64u : 128u, (uint32_t)R};
    const int ldS = bq_scales_ld(K);
    const uint64_t sdims[2] = {(uint64_t)(K / 32), (uint64_t)N};
    const uint64_t sstr[1] = {(uint64_t)ldS * 2};
    const uint32_t sbox[2] = {8, (uint32_t)R};
    if (!encode_tensor_map(&m->tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, W->codes, cdims, cstr,
                           cbox, low2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                           kPromoCodes) ||
        !encode_tensor_map(&m->tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W->scales, sdims, sstr,
                           sbox, CU_TENSOR_MAP_SWIZZLE_NONE, kPromoScales))
        return false;
    m->x = reinterpret_cast<const __half *>(x);
    m->y = y;
    m->N = N;
    m->K = K;
    m->B = B;
    m->cpb = (K + kChunkK - 1) / kChunkK;
    m->nbands = (N + R - 1) / R;
    m->chunk_base = 0;
    m->band_base = 0;
    m->epi = BQ_EPI_NONE;
    return true;
}

// An epilogue and the matrix it applies to: SwiGLU needs whole 16-row
// gate|up tiles.
bool epilogue_ok(int epi, int N)
{
    return epi == BQ_EPI_NONE || (epi == BQ_EPI_SWIGLU && N % 16 == 0);
}

void fill_stage(StageDesc *st, int mat_begin, int mat_end, long long T, int nbands, int wmax)
{
    st->mat_begin = mat_begin;
    st->mat_end = mat_end;
    st->T = (int)T;
    st->cpw = (int)std::max<long long>(1, (T + wmax - 1) / wmax);
    st->W = (int)((T + st->cpw - 1) / st->cpw);
    st->nbands = nbands;
}

// Q4 chunk height for one matrix launch.  A launch lasts as long as its
// busiest warp: its chunks, each a chain of dependent loads and mma, plus the
// sum of any band its range shares -- far dearer once some band's workers
// span CTAs (workspace partials and a GPU-scope arrival instead of shared
// memory).  32-row chunks take fewer instructions per weight; 16-row chunks
// halve a warp's unit of work and a band's split.  Both are estimated with a
// linear model fitted to launch-chain timings of Q4 shapes from 512 x 2048
// to 51200 x 5120 at B = 1 and 8 on a B200 (per warp: 0.19 per chunk + 1.15
// per 16-row tile, + 2.68 when a band crosses CTAs, + 0.35 per 16-row chunk
// at large B; microseconds), and the cheaper is taken.
int choose_q4_mt(long long N, long long K, int B, int cap_ctas)
{
    const long long cpb = (K + kChunkK - 1) / kChunkK;
    long long best = 0;
    int best_mt = 2;
    for (int mt = 2; mt >= 1; mt--) {
        const long long nbands = (N + 16 * mt - 1) / (16 * mt);
        const long long T = nbands * cpb;
        const long long wmax = std::min<long long>(cap_ctas, T) * kWarps;
        const long long cpw = std::max<long long>(1, (T + wmax - 1) / wmax);
        // Workers are numbered CTA-major, so CTA j starts at chunk
        // j * kWarps * cpw: some band crosses a CTA boundary unless every
        // boundary is a band boundary.
        const long long cta_chunks = kWarps * cpw;
        const bool crosses = cta_chunks < T && cta_chunks % cpb != 0;
        const long long cost = 19 * cpw + 115 * cpw * mt + (crosses ? 268 : 0) +
                               ((mt == 1 && B > 4) ? 35 * cpw : 0);
        if (mt == 2 || cost < best) {
            best = cost;
            best_mt = mt;
        }
    }
    return best_mt;
}

// Cluster size for a matrix launch whose bands would be summed across CTAs:
// the smallest C in {2, 4, 8} that makes every cluster boundary a band boundary
// (C * kWarps * cpw chunks a multiple of the chunks per band), so that every
// cross-CTA sum stays inside one cluster.  The grid shrinks to the CTAs that
// have chunks, rounded up to a multiple of C (no more than `cap`); the
// chunks per worker stay the same, and the device must hold all those
// clusters at once (`resident(C)`): a second wave would cost far more than
// the sums save.  (Clusters of 3, 5, 6 or 7, which the rule would also
// allow, measured slower than the workspace sums on full-device launches:
// 5 CTAs at 2 per SM leave SM slots that neither cluster can use.)  1 when
// the launch needs no cross-CTA sums or no C works.  *G becomes the grid of
// the chosen C.
template <class Resident>
int cluster_for(long long T, long long cpb, long long cpw, int *G, int cap, Resident resident)
{
    const long long cta_chunks = kWarps * cpw;
    if (!(cta_chunks < T && cta_chunks % cpb != 0))
        return 1;
    const long long busy = ((T + cpw - 1) / cpw + kWarps - 1) / kWarps;   // CTAs with chunks
    for (int c = 2; c <= kMaxCluster; c *= 2) {
        const long long Gc = (busy + c - 1) / c * c;
        if (Gc > cap)
            continue;
        const long long wmax = Gc * kWarps;
        if (std::max<long long>(1, (T + wmax - 1) / wmax) != cpw)
            continue;
        if ((c * cta_chunks) % cpb == 0 && (long long)resident(c) * c >= Gc) {
            *G = (int)Gc;
            return c;
        }
    }
    return 1;
}

// Launch geometry of one matrix: chunk height, the stream-K split, the grid
// and the cluster size.  `cap` is the CTA limit of a launch (2 per SM);
// `resident(mt, C)` the clusters of C CTAs the device holds at once.
struct Geometry {
    int mt;                 // 16-row m-tiles per chunk
    long long nbands, cpb, T;
    int cpw, G, C;
    bool crosses;           // some band's chunks span CTAs (before clusters)
};

template <class Resident>
Geometry matrix_geometry(int fmt, long long N, long long K, int B, int32_t rows_flag, int cap,
                         Resident resident)
{
    Geometry g;
    g.mt = fmt != 4 ? 1
                    : rows_flag == BQ_GEMV_ROWS16 ? 1
                    : rows_flag == BQ_GEMV_ROWS32 ? 2 : choose_q4_mt(N, K, B, cap);
    g.nbands = (N + 16 * g.mt - 1) / (16 * g.mt);
    g.cpb = (K + kChunkK - 1) / kChunkK;
    g.T = g.nbands * g.cpb;
    g.G = (int)std::min<long long>(cap, g.T);
    const long long wmax = (long long)g.G * kWarps;
    g.cpw = (int)std::max<long long>(1, (g.T + wmax - 1) / wmax);
    g.crosses = (long long)kWarps * g.cpw < g.T && ((long long)kWarps * g.cpw) % g.cpb != 0;
    const int mt = g.mt;
    g.C = BQ_CLUSTER_SUMS ? cluster_for(g.T, g.cpb, g.cpw, &g.G, cap,
                                        [&](int c) { return resident(mt, c); })
                          : 1;
    return g;
}

// Clusters of C CTAs of the cluster-sum kernel the device holds at once
// (cached per device and C as n + 1, 0 meaning not yet queried; atomic, since
// host threads may launch concurrently; 0 if the query fails).
template <int FMT, int MT>
int resident_clusters(int C)
{
    static std::atomic<int> cache[64][kMaxCluster + 1];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || C < 1 || C > kMaxCluster)
        return 0;
    const int known = cache[dev][C].load(std::memory_order_acquire);
    if (known > 0)
        return known - 1;
    int n = 0;
    if (prepare_kernel<FMT, kModeMatrix, MT, true>() == BQ_OK) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(C * kMaxCtas);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = launch_smem<FMT, MT>(1, 1, true);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, (const void *)stream_gemv_kernel<FMT, kModeMatrix, MT, true>,
                                           &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
        }
    }
    cache[dev][C].store(n + 1, std::memory_order_release);
    return n;
}

template <int FMT, int MT, bool CL>
int32_t gemv_launch_as(const KernelArgs &a0, int G, int C, void *stream)
{
    int32_t st = prepare_kernel<FMT, kModeMatrix, MT, CL>();
    if (st != BQ_OK)
        return st;
    KernelArgs a = a0;
    void *args[] = {&a};
    cudaError_t e = launch_pdl((const void *)stream_gemv_kernel<FMT, kModeMatrix, MT, CL>, dim3(G),
                               dim3(kThreads), launch_smem<FMT, MT>(1, 1, CL),
                               static_cast<cudaStream_t>(stream), args, C);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <int FMT, int MT>
int32_t gemv_launch(const bq_qmat *W, const uint16_t *x, int32_t B, void *y, int32_t epi,
                    int32_t flags, void *ws, int32_t *dev_status, void *stream, const Geometry &geo)
{
    KernelArgs a;
    memset(&a, 0, sizeof(a));
    if (!fill_matdesc(FMT, W, x, B, static_cast<float *>(y), &a.mat0, Fmt<FMT, MT>::kRows))
        return BQ_ERR_CUDA;
    if constexpr (FMT == 3 || FMT == 5 || FMT == 6) {
        // the top-bit plane: the last K/8 (Q3, Q5) or K/4 (Q6) bytes of each
        // row, after a first plane of K/4 (Q3) or K/2 bytes
        const int N = W->N, K = W->K;
        const int first = FMT == 3 ? K / 4 : K / 2;
        const int top = FMT == 6 ? K / 4 : K / 8;
        const uint64_t hdims[2] = {(uint64_t)top, (uint64_t)N};
        const uint64_t hstr[1] = {(uint64_t)(first + top)};
        const uint32_t hbox[2] = {(uint32_t)Fmt<FMT>::kTopRow, (uint32_t)Fmt<FMT>::kRows};
        if (!encode_tensor_map(&a.tm_codes_hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                               static_cast<const uint8_t *>(W->codes) + first, hdims, hstr, hbox,
                               CU_TENSOR_MAP_SWIZZLE_NONE, kPromoCodes))
            return BQ_ERR_CUDA;
    }
    a.mat0.epi = epi;
    a.prefill = (flags & BQ_GEMV_STATIC_WEIGHTS) ? 1 : 0;
    const long long T = (long long)a.mat0.cpb * a.mat0.nbands;
    const int G = geo.G, C = geo.C;
    a.wmax = G * kWarps;
    fill_stage(&a.stage0, 0, 1, T, a.mat0.nbands, a.wmax);
    if (a.stage0.cpw != geo.cpw)
        return BQ_ERR_CUDA;   // cannot happen: the geometry was computed for this shape
    a.n_stages = 1;
    a.counters = static_cast<int *>(ws);
    a.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + counters_bytes(a.mat0.nbands));
    a.status = dev_status;
    if (C > 1) {
        const int32_t st = gemv_launch_as<FMT, MT, true>(a, G, C, stream);
        if (st == BQ_OK)
            return st;
        // The device could not place the clusters: sum across CTAs through
        // the workspace instead (same results).
        (void)cudaGetLastError();
    }
    return gemv_launch_as<FMT, MT, false>(a, G, 1, stream);
}

template <int FMT>
int32_t gemv_impl(const bq_qmat *W, const uint16_t *x, int32_t B, void *y, int32_t epi,
                  int32_t flags, void *ws, size_t ws_bytes, int32_t *dev_status, void *stream)
{
    int32_t st = check_qmat(W);
    if (st != BQ_OK)
        return st;
    constexpr int32_t kKnown = BQ_GEMV_STATIC_WEIGHTS | BQ_GEMV_ROWS16 | BQ_GEMV_ROWS32;
    const int32_t rows = flags & (BQ_GEMV_ROWS16 | BQ_GEMV_ROWS32);
    if (!epilogue_ok(epi, W->N) || (flags & ~kKnown) != 0 ||
        rows == (BQ_GEMV_ROWS16 | BQ_GEMV_ROWS32) || (FMT != 4 && rows == BQ_GEMV_ROWS32) ||
        ((FMT == 6 || FMT == 2) && W->K % 64 != 0) || ((FMT == 5 || FMT == 3) && W->K % 128 != 0))
        return BQ_ERR_SHAPE;
    if (!x || !y || !ws)
        return BQ_ERR_NULL;
    if (B < 1 || B > 8)
        return BQ_ERR_BATCH;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws))
        return BQ_ERR_ALIGN;
    if (ws_bytes < bq_gemv_workspace_bytes(W->N, W->K))
        return BQ_ERR_WORKSPACE;
    const long long nbands = (W->N + 15) / 16;
    if (nbands * ((W->K + kChunkK - 1) / kChunkK) >= (1LL << 31))
        return BQ_ERR_SHAPE;
    const int cap = max_ctas();
    if (cap < 0)
        return BQ_ERR_CUDA;
    const Geometry geo = matrix_geometry(FMT, W->N, W->K, B, rows, cap, [](int mt, int c) {
        if constexpr (FMT != 4)
            return resident_clusters<FMT, 1>(c);
        else
            return mt == 1 ? resident_clusters<4, 1>(c) : resident_clusters<4, 2>(c);
    });
    if constexpr (FMT != 4) {
        return gemv_launch<FMT, 1>(W, x, B, y, epi, flags, ws, dev_status, stream, geo);
    } else {
        return geo.mt == 1 ? gemv_launch<4, 1>(W, x, B, y, epi, flags, ws, dev_status, stream, geo)
                           : gemv_launch<4, 2>(W, x, B, y, epi, flags, ws, dev_status, stream, geo);
    }
}

template <int FMT>
int32_t step_run_impl(const bq_step_info *info, const void *plan, void *ws, int32_t *dev_status,
                      void *stream, long long wait_cycles, int extra_arrivals)
{
    int32_t st = prepare_kernel<FMT, kModePlan>();
    if (st != BQ_OK)
        return st;
    KernelArgs a;
    memset(&a, 0, sizeof(a));
    const uint8_t *pb = static_cast<const uint8_t *>(plan);
    a.stages = reinterpret_cast<const StageDesc *>(pb + info->stages_off);
    a.mats = reinterpret_cast<const MatDesc *>(pb + info->mats_off);
    a.n_stages = info->n_stages;
    a.n_mats = info->n_mats;
    a.wmax = info->grid * kWarps;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    a.sync = reinterpret_cast<unsigned *>(wsb);
    a.counters = reinterpret_cast<int *>(wsb + kSyncBytes);
    a.partials = reinterpret_cast<float *>(wsb + kSyncBytes + counters_bytes(info->max_stage_bands));
    a.status = dev_status;
    a.wait_cycles = wait_cycles;
    a.extra_arrivals = extra_arrivals;
    void *args[] = {&a};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(info->grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = launch_smem<FMT>(info->n_stages, info->n_mats);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelExC(&cfg, (const void *)stream_gemv_kernel<FMT, kModePlan>, args);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_gemv_workspace_bytes(int32_t N, int32_t K)
{
    if (N < 1 || K < 32 || K % 32 != 0)
        return 0;
    const long long nbands = (N + 15) / 16;   // the finest band height of any format
    return counters_bytes(nbands) + kPartialsBytes;
}

extern "C" int32_t bq_gemv_geometry_of(int32_t fmt, int32_t N, int32_t K, int32_t B,
                                       int32_t flags, int32_t sm_count, bq_gemv_geometry *out)
{
    if (!out)
        return BQ_ERR_NULL;
    const int32_t rows = flags & (BQ_GEMV_ROWS16 | BQ_GEMV_ROWS32);
    constexpr int32_t kKnown = BQ_GEMV_STATIC_WEIGHTS | BQ_GEMV_ROWS16 | BQ_GEMV_ROWS32;
    if (fmt < 2 || fmt > 8 || fmt == 7 || N < 1 || K < 32 || K % 32 != 0 ||
        ((fmt == 6 || fmt == 2) && K % 64 != 0) || ((fmt == 5 || fmt == 3) && K % 128 != 0) ||
        (flags & ~kKnown) != 0 ||
        rows == (BQ_GEMV_ROWS16 | BQ_GEMV_ROWS32) || (fmt != 4 && rows == BQ_GEMV_ROWS32) ||
        sm_count < 0)
        return BQ_ERR_SHAPE;
    if (B < 1 || B > 8)
        return BQ_ERR_BATCH;
    Geometry g;
    if (sm_count > 0) {
        // a device of sm_count SMs that holds any cluster grid at once
        const int cap = std::min(BQ_MIN_BLOCKS * sm_count, kMaxCtas);
        g = matrix_geometry(fmt, N, K, B, rows, cap, [](int, int) { return kMaxCtas; });
    } else {
        const int cap = max_ctas();
        if (cap < 0)
            return BQ_ERR_CUDA;
        g = fmt == 4   ? matrix_geometry(4, N, K, B, rows, cap, [](int mt, int c) {
                return mt == 1 ? resident_clusters<4, 1>(c) : resident_clusters<4, 2>(c);
            })
            : fmt == 6 ? matrix_geometry(6, N, K, B, rows, cap,
                                         [](int, int c) { return resident_clusters<6, 1>(c); })
            : fmt == 5 ? matrix_geometry(5, N, K, B, rows, cap,
                                         [](int, int c) { return resident_clusters<5, 1>(c); })
            : fmt == 3 ? matrix_geometry(3, N, K, B, rows, cap,
                                         [](int, int c) { return resident_clusters<3, 1>(c); })
            : fmt == 2 ? matrix_geometry(2, N, K, B, rows, cap,
                                         [](int, int c) { return resident_clusters<2, 1>(c); })
                       : matrix_geometry(8, N, K, B, rows, cap,
                                         [](int, int c) { return resident_clusters<8, 1>(c); });
    }
    out->rows = 16 * g.mt;
    out->chunks = (int32_t)g.T;
    out->chunks_per_band = (int32_t)g.cpb;
    out->chunks_per_worker = g.cpw;
    out->grid = g.G;
    out->cluster = g.C;
    out->cross_cta_bands = g.crosses ? 1 : 0;
    out->reserved = 0;
    return BQ_OK;
}

extern "C" int32_t bq_gemv_q4(const bq_qmat *W, const uint16_t *x, int32_t B, float *y, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return gemv_impl<4>(W, x, B, y, BQ_EPI_NONE, 0, ws, ws_bytes, dev_status, stream);
}

extern "C" int32_t bq_gemv_q8(const bq_qmat *W, const uint16_t *x, int32_t B, float *y, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return gemv_impl<8>(W, x, B, y, BQ_EPI_NONE, 0, ws, ws_bytes, dev_status, stream);
}

extern "C" int32_t bq_gemv_ex(int32_t fmt, const bq_qmat *W, const uint16_t *x, int32_t B,
                              void *y, int32_t epilogue, int32_t flags, void *ws, size_t ws_bytes,
                              int32_t *dev_status, void *stream)
{
    if (fmt == 4)
        return gemv_impl<4>(W, x, B, y, epilogue, flags, ws, ws_bytes, dev_status, stream);
    if (fmt == 6)
        return gemv_impl<6>(W, x, B, y, epilogue, flags, ws, ws_bytes, dev_status, stream);
    if (fmt == 5)
        return gemv_impl<5>(W, x, B, y, epilogue, flags, ws, ws_bytes, dev_status, stream);
    if (fmt == 3)
        return gemv_impl<3>(W, x, B, y, epilogue, flags, ws, ws_bytes, dev_status, stream);
    if (fmt == 2)
        return gemv_impl<2>(W, x, B, y, epilogue, flags, ws, ws_bytes, dev_status, stream);
    if (fmt == 8)
        return gemv_impl<8>(W, x, B, y, epilogue, flags, ws, ws_bytes, dev_status, stream);
    return BQ_ERR_SHAPE;
}

// ------------------------------------------------------------ decode step --
extern "C" size_t bq_step_plan_bytes(int32_t n_mats)
{
    if (n_mats < 1)
        return 0;
    return align_up(sizeof(PlanHeader), 64) + align_up((size_t)n_mats * sizeof(StageDesc), 64) +
           (size_t)n_mats * sizeof(MatDesc);
}

extern "C" int32_t bq_step_plan(int32_t fmt, const bq_step_mat *mats, int32_t n_mats, void *plan,
                                size_t plan_bytes, bq_step_info *info)
{
    if (!mats || !plan || !info)
        return BQ_ERR_NULL;
    if ((fmt != 4 && fmt != 8) || n_mats < 1 || n_mats > kMaxPlanMats)
        return BQ_ERR_SHAPE;
    if (plan_bytes < bq_step_plan_bytes(n_mats))
        return BQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(plan) & 63u) != 0)
        return BQ_ERR_ALIGN;
    for (int i = 0; i < n_mats; i++) {
        const int32_t st = check_qmat(&mats[i].W);
        if (st != BQ_OK)
            return st;
        if (!mats[i].x || !mats[i].y)
            return BQ_ERR_NULL;
        if (mats[i].B < 1 || mats[i].B > 8)
            return BQ_ERR_BATCH;
        if (mats[i].stage < 0 || !epilogue_ok(mats[i].epilogue, mats[i].W.N))
            return BQ_ERR_SHAPE;
        if (!aligned16(mats[i].x) || !aligned16(mats[i].y))
            return BQ_ERR_ALIGN;
    }
    int32_t st = fmt == 4 ? prepare_kernel<4, kModePlan>() : prepare_kernel<8, kModePlan>();
    if (st != BQ_OK)
        return st;
    // Co-residency: every CTA of the grid must fit on the device at once.
    int occ = 0;
    const void *kfn = fmt == 4 ? (const void *)stream_gemv_kernel<4, kModePlan>
                               : (const void *)stream_gemv_kernel<8, kModePlan>;
    // (n_stages <= n_mats, so sizing the cache for n_mats stages is an upper bound)
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &occ, kfn, kThreads,
            fmt == 4 ? launch_smem<4>(n_mats, n_mats) : launch_smem<8>(n_mats, n_mats)) !=
            cudaSuccess ||
        occ < 1)
        return BQ_ERR_CUDA;
    const int sms = device_sm_count();
    if (sms <= 0)
        return BQ_ERR_CUDA;
    const int G = std::min(std::min(occ, BQ_MIN_BLOCKS) * sms, kMaxCtas);
    const int wmax = G * kWarps;

    std::vector<int> order(n_mats);
    for (int i = 0; i < n_mats; i++)
        order[i] = i;
    std::stable_sort(order.begin(), order.end(),
                     [&](int p, int q) { return mats[p].stage < mats[q].stage; });
    std::vector<MatDesc> md(n_mats);
    std::vector<StageDesc> sd;
    long long max_bands = 1;
    for (int i = 0; i < n_mats;) {
        const int s = mats[order[i]].stage;
        int j = i;
        long long T = 0, bands = 0;
        while (j < n_mats && mats[order[j]].stage == s) {
            const bq_step_mat &m = mats[order[j]];
            if (!fill_matdesc(fmt, &m.W, m.x, m.B, static_cast<float *>(m.y), &md[j]))
                return BQ_ERR_CUDA;
            md[j].epi = m.epilogue;
            md[j].chunk_base = (int)T;
            md[j].band_base = (int)bands;
            T += (long long)md[j].cpb * md[j].nbands;
            bands += md[j].nbands;
            if (T >= (1LL << 31))
                return BQ_ERR_SHAPE;
            j++;
        }
        StageDesc sdesc;
        fill_stage(&sdesc, i, j, T, (int)bands, wmax);
        sd.push_back(sdesc);
        max_bands = std::max(max_bands, bands);
        i = j;
    }
    PlanHeader h;
    memset(&h, 0, sizeof(h));
    h.magic = kPlanMagic;
    h.fmt = fmt;
    h.n_mats = n_mats;
    h.n_stages = (int)sd.size();
    h.grid = G;
    h.max_stage_bands = (int)max_bands;
    h.stages_off = align_up(sizeof(PlanHeader), 64);
    h.mats_off = h.stages_off + align_up((size_t)n_mats * sizeof(StageDesc), 64);
    std::vector<uint8_t> host(h.mats_off + (size_t)n_mats * sizeof(MatDesc), 0);
    memcpy(host.data(), &h, sizeof(h));
    memcpy(host.data() + h.stages_off, sd.data(), sd.size() * sizeof(StageDesc));
    memcpy(host.data() + h.mats_off, md.data(), (size_t)n_mats * sizeof(MatDesc));
    if (cudaMemcpy(plan, host.data(), host.size(), cudaMemcpyHostToDevice) != cudaSuccess)
        return BQ_ERR_CUDA;
    info->fmt = fmt;
    info->n_mats = n_mats;
    info->n_stages = h.n_stages;
    info->grid = G;
    info->max_stage_bands = (int)max_bands;
    info->stages_off = h.stages_off;
    info->mats_off = h.mats_off;
    info->ws_bytes = kSyncBytes + counters_bytes(max_bands) + kPartialsBytes;
    return BQ_OK;
}

extern "C" int32_t bq_step_run_ex(const bq_step_info *info, const void *plan, void *ws,
                                  size_t ws_bytes, const bq_step_wait *wait, int32_t *dev_status,
                                  void *stream)
{
    if (!info || !plan || !ws)
        return BQ_ERR_NULL;
    if ((info->fmt != 4 && info->fmt != 8) || info->n_stages < 1 || info->grid < 1)
        return BQ_ERR_SHAPE;
    if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(plan) & 63u) != 0)
        return BQ_ERR_ALIGN;
    if (ws_bytes < info->ws_bytes)
        return BQ_ERR_WORKSPACE;
    long long cycles = kWaitCycles;
    int extra = 0;
    if (wait) {
        if (wait->wait_cycles < 0 || wait->extra_arrivals < 0 || wait->extra_arrivals > 1024)
            return BQ_ERR_SHAPE;
        if (wait->wait_cycles > 0)
            cycles = std::min<long long>(wait->wait_cycles, kWaitCycles);   // (the warps' own limit)
        extra = wait->extra_arrivals;
    }
    return info->fmt == 4 ? step_run_impl<4>(info, plan, ws, dev_status, stream, cycles, extra)
                          : step_run_impl<8>(info, plan, ws, dev_status, stream, cycles, extra);
}

extern "C" int32_t bq_step_run(const bq_step_info *info, const void *plan, void *ws,
                               size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return bq_step_run_ex(info, plan, ws, ws_bytes, nullptr, dev_status, stream);
}

// ------------------------------------------------------- routed experts --
extern "C" size_t bq_moe_workspace_bytes(int32_t N, int32_t K, int32_t B, int32_t topk, int32_t E)
{
    if (N < 1 || K < 32 || K % 32 != 0 || B < 1 || B > 8 || topk < 1 || B * topk > kMaxSlots ||
        E < 1 || E > 65535)
        return 0;
    const long long nbands = (N + 15) / 16;   // the finest band height (16-row chunks)
    return counters_bytes(nbands * B * topk) + kPartialsBytes +
           align_up((size_t)B * topk * N * sizeof(float), 256);
}

extern "C" int32_t bq_moe_gemv_q4(const bq_qmat *Wstack, int32_t E, int64_t codes_stride,
                                  int64_t scales_stride, const uint16_t *x, int32_t x_per_slot,
                                  const int32_t *expert_idx, const float *route_w, int32_t B,
                                  int32_t topk, float *y, void *ws, size_t ws_bytes,
                                  int32_t *dev_status, void *stream)
{
    return bq_moe_gemv_ex(Wstack, E, codes_stride, scales_stride, x, x_per_slot, expert_idx,
                          route_w, B, topk, y, BQ_EPI_NONE, ws, ws_bytes, dev_status, stream);
}

namespace bq {
namespace {
template <int MT>
int32_t moe_launch(const bq_qmat *Wstack, int32_t E, int64_t codes_stride, int64_t scales_stride,
                   const uint16_t *x, int32_t x_per_slot, const int32_t *expert_idx,
                   const float *route_w, int32_t B, int32_t topk, void *y, int32_t epilogue,
                   void *ws, int32_t *dev_status, void *stream, int G)
{
    constexpr int R = Fmt<4, MT>::kRows;
    const int N = Wstack->N, K = Wstack->K, ldS = bq_scales_ld(K);
    const long long nbands = (N + R - 1) / R;
    const long long cpb = (K + kChunkK - 1) / kChunkK;
    int32_t st = prepare_kernel<4, kModeMoE, MT>();
    if (st != BQ_OK)
        return st;

    KernelArgs a;
    memset(&a, 0, sizeof(a));
    const uint64_t cdims[3] = {(uint64_t)(K / 2), (uint64_t)N, (uint64_t)E};
    const uint64_t cstr[2] = {(uint64_t)(K / 2), (uint64_t)codes_stride};
    const uint32_t cbox[3] = {128, (uint32_t)R, 1};
    const uint64_t sdims[3] = {(uint64_t)(K / 32), (uint64_t)N, (uint64_t)E};
    const uint64_t sstr[2] = {(uint64_t)ldS * 2, (uint64_t)scales_stride * 2};
    const uint32_t sbox[3] = {8, (uint32_t)R, 1};
    if (!encode_tensor_map(&a.mat0.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, Wstack->codes,
                           cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_128B, kPromoCodes) ||
        !encode_tensor_map(&a.mat0.tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, Wstack->scales,
                           sdims, sstr, sbox, CU_TENSOR_MAP_SWIZZLE_NONE, kPromoScales))
        return BQ_ERR_CUDA;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    float *slot_buf = reinterpret_cast<float *>(wsb + counters_bytes(nbands * B * topk) + kPartialsBytes);
    a.mat0.x = reinterpret_cast<const __half *>(x);
    a.mat0.y = route_w ? slot_buf : static_cast<float *>(y);
    a.mat0.epi = epilogue;
    a.mat0.N = N;
    a.mat0.K = K;
    a.mat0.B = B;
    a.mat0.cpb = (int)cpb;
    a.mat0.nbands = (int)nbands;
    a.wmax = G * kWarps;
    a.n_stages = 1;
    a.counters = reinterpret_cast<int *>(wsb);
    a.partials = reinterpret_cast<float *>(wsb + counters_bytes(nbands * B * topk));
    a.status = dev_status;
    a.E = E;
    a.topk = topk;
    a.x_per_slot = x_per_slot ? 1 : 0;
    a.idx = expert_idx;
    void *args[] = {&a};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_pdl((const void *)stream_gemv_kernel<4, kModeMoE, MT>, dim3(G),
                               dim3(kThreads), launch_smem<4, MT>(1, 1), s, args);
    if (e != cudaSuccess)
        return BQ_ERR_CUDA;
    if (route_w) {
        float *sb = slot_buf;
        int Bv = B, tk = topk, Nv = N, Ev = E;
        float *yc = static_cast<float *>(y);
        void *cargs[] = {(void *)&sb, (void *)&expert_idx, (void *)&route_w, &Bv, &tk, &Nv, &Ev, &yc};
        int cg = (B * N + 255) / 256;
        cg = std::max(1, std::min(cg, 4 * std::max(1, device_sm_count())));
        e = launch_pdl((const void *)moe_combine_kernel, dim3(cg), dim3(256), 0, s, cargs);
        if (e != cudaSuccess)
            return BQ_ERR_CUDA;
    }
    return BQ_OK;
}
}  // namespace
}  // namespace bq

extern "C" int32_t bq_moe_gemv_ex(const bq_qmat *Wstack, int32_t E, int64_t codes_stride,
                                  int64_t scales_stride, const uint16_t *x, int32_t x_per_slot,
                                  const int32_t *expert_idx, const float *route_w, int32_t B,
                                  int32_t topk, void *y, int32_t epilogue, void *ws,
                                  size_t ws_bytes, int32_t *dev_status, void *stream)
{
    int32_t st = check_qmat(Wstack);
    if (st != BQ_OK)
        return st;
    if (!epilogue_ok(epilogue, Wstack->N) || (epilogue == BQ_EPI_SWIGLU && route_w))
        return BQ_ERR_SHAPE;
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
    const long long cpb = (K + kChunkK - 1) / kChunkK;
    if ((long long)B * topk * ((N + 15) / 16) * cpb >= (1LL << 31))
        return BQ_ERR_SHAPE;
    const int G = max_ctas();
    if (G < 0)
        return BQ_ERR_CUDA;
    // Chunk height as for one matrix, over the rows of the routed experts'
    // pieces (at most B * topk of them, one per distinct expert and up to 8
    // slots each).
    const long long pieces = std::min<long long>((long long)B * topk, E);
    const int mt = choose_q4_mt((long long)N * pieces, K, 1, G);
    return mt == 1 ? moe_launch<1>(Wstack, E, codes_stride, scales_stride, x, x_per_slot, expert_idx,
                                   route_w, B, topk, y, epilogue, ws, dev_status, stream, G)
                   : moe_launch<2>(Wstack, E, codes_stride, scales_stride, x, x_per_slot, expert_idx,
                                   route_w, B, topk, y, epilogue, ws, dev_status, stream, G);
}


// ------------------------------------------------- Q4 GEMV without workspace --
// Some callers cannot hand the library a workspace: code embedded in a host
// framework that owns every device allocation, or a latency-critical decode
// loop that must never call cudaMalloc (which can synchronise the device).
// bq_gemv_q4_noalloc serves them with the scratch the split-band sums need
// (arrival counters + partial sums) held in one fixed device array below.
// That array is part of the loaded library: every GPU that loads it keeps
// kNoAllocScratchBytes reserved until the process exits.
namespace bq {
namespace {
constexpr int kNoAllocMaxCtas = 320;                     // CTAs of one launch at most
constexpr long long kNoAllocMaxRows = 1LL << 20;         // N limit of this entry point
constexpr size_t kNoAllocCounterBytes = (size_t)(kNoAllocMaxRows / 16) * sizeof(int);
constexpr size_t kNoAllocPartialBytes =
    (size_t)kNoAllocMaxCtas * 2 * Fmt<4>::kMT * 32 * sizeof(float4);
constexpr size_t kNoAllocScratchBytes = kNoAllocCounterBytes + kNoAllocPartialBytes;
// The size the header states (262,144 bytes of counters + 655,360 of partials).
static_assert(kNoAllocScratchBytes == 917504, "the documented size of the no-allocation scratch");
}  // namespace
}  // namespace bq

static __device__ __align__(256) uint8_t g_bq_noalloc_scratch[bq::kNoAllocScratchBytes];

namespace bq {
namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64];   // device address of the scratch array, per device

// Device address of the scratch array on the current device.  The host-side
// name g_bq_noalloc_scratch is only a stand-in, never a device address, so it
// is looked up once per device (with that device current) and cached.
void *noalloc_scratch(int32_t *err)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *err = BQ_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bq_noalloc_scratch) != cudaSuccess || !p) {
            *err = BQ_ERR_CUDA;
            return nullptr;
        }
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace
}  // namespace bq

extern "C" int32_t bq_gemv_q4_noalloc(const bq_qmat *W, const uint16_t *x, int32_t B, float *y,
                                      int32_t *dev_status, void *stream)
{
    int32_t st = check_qmat(W);
    if (st != BQ_OK)
        return st;
    if (!x || !y)
        return BQ_ERR_NULL;
    if (B < 1 || B > 8)
        return BQ_ERR_BATCH;
    if (!aligned16(x) || !aligned16(y))
        return BQ_ERR_ALIGN;
    if (W->N > kNoAllocMaxRows)
        return BQ_ERR_WORKSPACE;   // more rows than the fixed scratch covers
    const long long nbands16 = (W->N + 15) / 16;
    if (nbands16 * ((W->K + kChunkK - 1) / kChunkK) >= (1LL << 31))
        return BQ_ERR_SHAPE;
    st = prepare_kernel<4, kModeMatrix>();
    if (st != BQ_OK)
        return st;
    int32_t err = BQ_OK;
    uint8_t *scratch = static_cast<uint8_t *>(noalloc_scratch(&err));
    if (!scratch)
        return err;

    KernelArgs a;
    memset(&a, 0, sizeof(a));
    if (!fill_matdesc(4, W, x, B, y, &a.mat0))
        return BQ_ERR_CUDA;
    const long long T = (long long)a.mat0.cpb * a.mat0.nbands;
    const int cap = max_ctas();
    if (cap < 0)
        return BQ_ERR_CUDA;
    const int G = (int)std::min<long long>(std::min(cap, kNoAllocMaxCtas), T);
    a.wmax = G * kWarps;
    fill_stage(&a.stage0, 0, 1, T, a.mat0.nbands, a.wmax);
    a.n_stages = 1;
    a.counters = reinterpret_cast<int *>(scratch);
    a.partials = reinterpret_cast<float *>(scratch + kNoAllocCounterBytes);
    a.status = dev_status;
    // The array keeps whatever the previous call left; the band counters
    // must start at zero, so clear them on this call's stream first.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(a.counters, 0, (size_t)a.mat0.nbands * sizeof(int), s) != cudaSuccess)
        return BQ_ERR_CUDA;
    void *args[] = {&a};
    cudaError_t e = launch_pdl((const void *)stream_gemv_kernel<4, kModeMatrix>, dim3(G),
                               dim3(kThreads), launch_smem<4>(1, 1), s, args);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

extern "C" int32_t bq_gemv_q4_noalloc_scratch(void **dev_ptr, size_t *bytes)
{
    if (!dev_ptr || !bytes)
        return BQ_ERR_NULL;
    int32_t err = BQ_OK;
    void *p = noalloc_scratch(&err);
    if (!p)
        return err;
    *dev_ptr = p;
    *bytes = kNoAllocScratchBytes;
    return BQ_OK;
}
