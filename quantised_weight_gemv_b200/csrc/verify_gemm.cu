// verify_gemm.cu -- the batched-verification GEMM over block-quantised
// weights (Q4 / Q8, batch 1..32) on the 5th-generation tensor cores (sm_100a).
//
// The pages name speculative decoding as the way past the decode bandwidth
// ceiling: the drafted tokens are checked in one batched verification step
// whose matrix products are compute-shaped and suit the tensor-core path
// (romaanj.github.io review of the M5 follow-up paper, "Future work").  Such a
// step multiplies the same packed weights by a small batch of activation
// vectors, B = 8..32: y[b][n] = sum_k deq(W)[n][k] x[b][k], with
// deq(W) = d (q - z) per 32-weight block, the decode GEMV's operation at a
// wider batch.  At B = 32 a Q4 weight carries 64 flop for 0.5625 bytes, so the
// legacy mma.sync path of the decode GEMV (whose per-column tiles grow with B)
// would be bound by its tensor pipe long before HBM; tcgen05.mma with the
// batch as the MMA's N dimension does the whole batch in one instruction.
//
// Tile: 128 weight rows x all B columns, accumulated in tensor memory (TMEM:
// 128 lanes = rows, NB = 16 or 32 fp32 columns = batch).  Work unit: one
// tile x 256 weights of K.  Units are numbered tile-major (K fastest) and
// split into one contiguous range per CTA (one CTA per SM, stream-K), so every
// SM streams the same number of weight bytes; a tile whose units span several
// CTAs is summed deterministically through the workspace (last arriver adds
// the CTA partials in CTA order).
//
// Warp roles (16 warps):
//   warp 0      TMA of a unit's packed codes (128-byte swizzle), scales and
//               activations x (K-major, 128-byte swizzle: the layout the
//               MMA's B descriptor reads; rows >= B zero-filled) into a ring
//               of 4-6 unit slots, so x arrives units ahead of its MMAs;
//   warp 1      allocates TMEM (512 columns: two accumulators and a ring of
//               6 dequantised A sub-stages), and one thread issues the MMAs:
//               per unit one wait (every dequant warp has stored the unit's
//               A), then per 128-weight sub-stage 8 x tcgen05.mma (M 128, N
//               NB, K 16, fp16 in, fp32 accumulation) with A read from TMEM
//               and x from a shared-memory descriptor, and tcgen05.commit to
//               free the A slot (after a unit's last one, also its ring slot);
//   warps 2-3   row shifts (below) of each segment, a few segments ahead;
//   warps 4-7   epilogue: tcgen05.ld of the accumulator, one thread per row;
//   warps 8-15  dequantisation: warp w serves TMEM lanes 32 (w % 4) .. + 31
//               (rows) and one half of each sub-stage; a thread turns two
//               blocks of its row (32 or 64 code bytes and two fp16 scales)
//               into 64 fp16 weights d (q - z) 2^s and writes them as 32 TMEM
//               columns with tcgen05.st.  At the start they also compute the
//               first two segments' row shifts, one row each.
// A lives in TMEM, not shared memory: a 128 x 16 fp16 A operand is 4 KB, and
// reading it from shared memory for every K16 step (plus writing it there
// first) would need more shared-memory bandwidth than the Q4 stream leaves.
// Measured on B200: a tcgen05.mma of M 128 x N <= 64 x K 16 takes a fixed
// ~70-130 cycles of the tensor pipe whatever N (N = 256 takes ~130), so the
// MMA side caps a Q4 verification step near 0.5 of HBM; an mbarrier wait in
// the issuing thread stalls the pipe for its whole latency (the MMA queue is
// short), hence one wait per 16 MMAs.

// Rounding.  The decode GEMV keeps codes exact and scales each block's sum;
// a tile accumulated over many blocks cannot, so the A tile holds each weight
// rounded once to fp16: relative error <= 2^-11, inside the decode tolerance
// (1e-3 * sum |w x|).  To keep that bound for any scale, each row's values are
// multiplied by a power of two 2^s chosen from the largest scale of the row in
// the CTA's K range (the largest |d (q - z)| 2^s lies in [2^14, 2^15)), and
// the epilogue multiplies by 2^-s: no overflow, and subnormal fp16 only for
// blocks 2^28 times smaller than the row's largest.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {
namespace vg {

#ifndef BQ_VERIFY_DQ_GROUPS
#define BQ_VERIFY_DQ_GROUPS 1
#endif
constexpr int kDqGroups = BQ_VERIFY_DQ_GROUPS;   // dequant warp groups (8 warps each), alternate sub-stages
constexpr int kThreads = (8 + 8 * kDqGroups) * 32;
constexpr int TM = 128;                 // rows per tile (MMA M)
constexpr int kUnitK = 256;             // weights of K per unit
constexpr int kSubK = 128;              // weights of K per sub-stage (one hand-off to the MMA thread)
constexpr int kXK = 64;                 // weights of K per x tile (one 128-byte swizzle row of fp16)
constexpr int AS = 6;                   // A sub-stage slots in tensor memory (3 units)
constexpr int kAccCols = 64;            // TMEM columns of the two accumulators (up to 32 each)
constexpr int kACols = kSubK / 2;       // TMEM columns of one A sub-stage (two fp16 a column)
constexpr int kTmemCols = 512;
static_assert(kAccCols + AS * kACols <= kTmemCols, "accumulators and the A ring fit in TMEM");
constexpr int kShiftRing = 4;           // row shifts of the last 4 segments
constexpr int kMaxCtas = 512;
constexpr int kScaleBytes = TM * 16;    // 8 fp16 per row per unit
constexpr int kDequantWarp0 = 8;
constexpr int kEpiWarp0 = 4;

template <int FMT> struct VFmt;
template <> struct VFmt<4> {
    static constexpr int kCodeBytes = TM * 128;   // one 128 x 128-byte box
};
template <> struct VFmt<8> {
    static constexpr int kCodeBytes = TM * 256;   // two 128 x 128-byte boxes
};

// A unit's ring slot: codes, then x (4 sub-tiles of NB rows x 64 fp16), then
// scales.
template <int FMT, int NB>
__host__ __device__ constexpr int slot_bytes()
{
    return VFmt<FMT>::kCodeBytes + 4 * NB * 128 + kScaleBytes;
}

// Unit slots of the ring: as many as ~200 KB of shared memory holds (4 to 6).
template <int FMT, int NB>
__host__ __device__ constexpr int ring_slots()
{
    return (200 * 1024) / slot_bytes<FMT, NB>() < 6 ? (200 * 1024) / slot_bytes<FMT, NB>() : 6;
}

template <int FMT, int NB>
constexpr size_t smem_bytes()
{
    return 1024 + (size_t)ring_slots<FMT, NB>() * slot_bytes<FMT, NB>() + 1024;
}

// Per-tile partial sums through the workspace: [CTA][slot 0 / 1][TM][32] fp32.
constexpr size_t kPartBytesPerCta = 2 * TM * 32 * sizeof(float);

struct Args {
    CUtensorMap tm_codes;    // Q4: (K/2, N) bytes; Q8: (K, N) bytes; box 128 x 128, SW128
    CUtensorMap tm_scales;   // (K/32, N) u16, box 8 x 128
    CUtensorMap tm_x;        // (K, B) f16, box 64 x NB, SW128
    const uint16_t *scales;  // the scale plane (pre-pass reads it directly)
    float *y;                // [B][N]
    int N, K, B, ldS;
    int ntiles, KU, U, G;    // tiles, units per tile, units, CTAs
    int *counters;           // [ntiles], zero on entry and exit
    float *partials;         // [G][2][TM][32]
    int *status;
};

// ----------------------------------------------------------- tcgen05 ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (fp16 x fp16 -> fp32).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive (once) on an mbarrier when every tcgen05 operation this thread
// issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart (stride
// dimension offset), start address 16-byte granular; descriptor version 1,
// layout type 2 (SWIZZLE_128B).  The leading-dimension offset is unused by
// swizzled K-major layouts (set to 1).
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// 32 lanes x N consecutive fp32 columns of TMEM into registers (this warp's
// lane quarter).
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++)
        v[i] = __uint_as_float(r[i]);
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++)
        v[i] = __uint_as_float(r[i]);
}

// 32 consecutive 32-bit TMEM columns of this thread's lane (32x32b shape: a
// warp writes its 32 lanes); asynchronous: tmem_wait_st() waits for the
// warp's stores.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31, %32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
          "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
          "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
          "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
          "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16: A's row m is TMEM lane m,
// its K elements two to a 32-bit column.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ int ld_acquire_gpu_int(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t hadd2_u(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// fp16 pairs: 0x6400 | byte is the fp16 value 1024 + byte, exactly.
constexpr uint32_t kMagic = 0x64646464u;
constexpr uint32_t kNeg1032 = 0xE408E408u;   // -1032 (Q4: 1024 + zero point 8)
constexpr uint32_t kNeg72 = 0xD480D480u;     // -72   (Q4 high nibble: 64 + 8)
constexpr uint32_t kSixteenth = 0x2C002C00u; // 1/16
constexpr uint32_t kNeg1152 = 0xE480E480u;   // -1152 (Q8: 1024 + 128)

// Q4: the 32 weights of one block (16 code bytes; byte i holds element i in
// its low and element i + 16 in its high nibble) as fp16 (q - 8) * ds, two a
// register in element order: o[c] = elements (2c, 2c + 1).  (1024 + nibble)
// - 1032 and (1024 + 16 nibble) / 16 - 72 are exact; the product by ds is the
// one rounding.
__device__ __forceinline__ void dequant_q4_block(uint4 c, uint32_t ds2, uint32_t (&o)[16])
{
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t p0 = prmt(w[i], kMagic, 0x4140);   // bytes 4i, 4i+1
        const uint32_t p1 = prmt(w[i], kMagic, 0x4342);   // bytes 4i+2, 4i+3
        o[2 * i] = hmul2_u(hadd2_u(p0 & 0xFF0FFF0Fu, kNeg1032), ds2);              // elements 4i, 4i+1
        o[2 * i + 1] = hmul2_u(hadd2_u(p1 & 0xFF0FFF0Fu, kNeg1032), ds2);          // 4i+2, 4i+3
        o[8 + 2 * i] = hmul2_u(hfma2_u(p0 & 0xFFF0FFF0u, kSixteenth, kNeg72), ds2);     // 16+4i, +1
        o[8 + 2 * i + 1] = hmul2_u(hfma2_u(p1 & 0xFFF0FFF0u, kSixteenth, kNeg72), ds2); // 16+4i+2, +3
    }
}

// Q8: 16 signed code bytes (elements e .. e+15) as fp16 q * ds into o[0..7]
// in element order: (byte ^ 0x80) = q + 128, (1024 + q + 128) - 1152 = q
// exactly.
__device__ __forceinline__ void dequant_q8_half(uint4 c, uint32_t ds2, uint32_t *o)
{
    const uint32_t w[4] = {c.x ^ 0x80808080u, c.y ^ 0x80808080u, c.z ^ 0x80808080u, c.w ^ 0x80808080u};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        o[2 * i] = hmul2_u(hadd2_u(prmt(w[i], kMagic, 0x4140), kNeg1152), ds2);
        o[2 * i + 1] = hmul2_u(hadd2_u(prmt(w[i], kMagic, 0x4342), kNeg1152), ds2);
    }
}

// The CTA owning unit x under the balanced split of U units over G CTAs
// (CTA c owns [floor(c U / G), floor((c + 1) U / G))).
__device__ __forceinline__ int owner_of(long long x, int U, int G)
{
    return (int)(((x + 1) * G - 1) / U);
}

template <int FMT, int NB>
__global__ void __launch_bounds__(kThreads, 1) verify_gemm_kernel(const __grid_constant__ Args a)
{
    using VF = VFmt<FMT>;
    constexpr int CS = ring_slots<FMT, NB>();
    constexpr int CB = VF::kCodeBytes;
    constexpr int XB = NB * 128;   // x bytes per sub-stage
    constexpr int SLOT = slot_bytes<FMT, NB>();
    extern __shared__ uint8_t smem_raw[];
    __shared__ alignas(8) uint64_t bar_cfull[CS], bar_cempty[CS], bar_ufull[AS], bar_aempty[AS],
        bar_accfull[2], bar_accempty[2], bar_shift[kShiftRing],
        bar_shift_free[kShiftRing], bar_done, bar_pre,
        bar_epi_a, bar_epi_b;
    __shared__ uint32_t tmem_base_s;
    __shared__ int shift_s[kShiftRing][TM];
    __shared__ int epi_old;
    __shared__ int abort_s;

    uint8_t *sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t ring_s = smem_u32(sbase);                 // CS unit slots (1024-aligned)
    static_assert(SLOT % 1024 == 0, "unit slots keep the 1024-byte alignment of the swizzled boxes");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int u0 = (int)((long long)cta * a.U / a.G), u1 = (int)((long long)(cta + 1) * a.U / a.G);

    if (threadIdx.x == 0) {
        for (int i = 0; i < CS; i++) {
            mbar_init(smem_u32(&bar_cfull[i]), 1);
            mbar_init(smem_u32(&bar_cempty[i]), 8 * kDqGroups + 1);   // every dequant warp + the MMAs' commit
        }
        for (int i = 0; i < AS; i++) {
            mbar_init(smem_u32(&bar_ufull[i]), 8 * kDqGroups);   // every dequant warp, once a unit
            mbar_init(smem_u32(&bar_aempty[i]), 1);          // tcgen05.commit
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(smem_u32(&bar_accfull[i]), 1);         // tcgen05.commit
            mbar_init(smem_u32(&bar_accempty[i]), 4);        // the 4 epilogue warps
        }
        for (int i = 0; i < kShiftRing; i++) {
            mbar_init(smem_u32(&bar_shift[i]), 2);           // the row-shift warps 2-3
            mbar_init(smem_u32(&bar_shift_free[i]), 4 + 8 * kDqGroups);   // epilogue + dequant warps
        }
        mbar_init(smem_u32(&bar_done), 1);
        mbar_init(smem_u32(&bar_pre), 8 * kDqGroups);        // dequant warps: first two segments' shifts
        mbar_init(smem_u32(&bar_epi_a), 128);                // the epilogue's split-tile handshake
        mbar_init(smem_u32(&bar_epi_b), 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_base_s), kTmemCols);       // accumulators + the A ring (1 CTA / SM)
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    // Programmatic dependent launch: let the next kernel on the stream get
    // scheduled, and touch no global memory before the previous one has
    // completed.
    pdl_launch_dependents();
    pdl_wait();

    // Failure path: a bounded wait ran out -- report, and make every role stop.
    auto fail = [&]() {
        if (a.status)
            atomicOr(a.status, kStatusTimeout);
        *(volatile int *)&abort_s = 1;
    };
    auto aborted = [&]() { return *(volatile int *)&abort_s != 0; };
    auto wait = [&](uint64_t &bar, uint32_t parity) -> bool {
        if (mbar_wait_bounded(smem_u32(&bar), parity))
            return true;
        fail();
        return false;
    };
    // Sub-stages of unit u (the last unit of a row may be short).
    auto nsub = [&](int u) {
        const int ku = u % a.KU;
        return min(kUnitK / kSubK, (a.K - ku * kUnitK + kSubK - 1) / kSubK);
    };

    // Largest |scale| (fp16 bits without the sign) of one row of a tile
    // over n units from ub (16 bytes a unit), sixteen loads in flight.
    auto row_scale_max = [&](int tile, int ub, int n, int r) -> unsigned {
        const int row = tile * TM + r;
        unsigned m = 0u;
        if (row >= a.N)
            return m;
        const uint16_t *srow = a.scales + (size_t)row * a.ldS;
        for (int k0 = 0; k0 < n; k0 += 16) {
            uint4 v[16];
#pragma unroll
            for (int k = 0; k < 16; k++)
                v[k] = k0 + k < n ? __ldg(reinterpret_cast<const uint4 *>(srow + (size_t)((ub + k0 + k) % a.KU) * 8))
                                  : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int k = 0; k < 16; k++) {
                const uint32_t sv[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                for (int e = 0; e < 4; e++)
                    m = max(m, max(sv[e] & 0x7FFFu, (sv[e] >> 16) & 0x7FFFu));
            }
        }
        return m;
    };
    // The row shift s for a row whose largest scale has fp16 bits m: the
    // largest |d (q - z)| (8 dmax for Q4, 127 dmax for Q8) times 2^s lands
    // in [2^14, 2^15).
    auto shift_of = [](unsigned m) -> int {
        m = min(m, 0x7BFFu);                                  // largest finite fp16
        const float top = __half2float(__ushort_as_half((unsigned short)m)) * (FMT == 4 ? 8.0f : 127.0f);
        return top > 0.f ? 141 - ((__float_as_int(top) >> 23) & 0xFF) : 0;
    };
    // The CTA's segments (its units of one tile each) in processing order.
    // A range that ends inside a tile shares that tile with the next CTA,
    // which does the tile's other units at the start of its range; doing
    // this CTA's part first too lets the tile's cross-CTA sum happen early,
    // under later units, instead of at the end of both CTAs.  So the last
    // segment goes first when it is a partial tile; the others keep order.
    const int seg_t0 = u0 / a.KU;
    const int seg_n = (u1 - 1) / a.KU - seg_t0 + 1;
    const bool seg_rot = seg_n > 1 && u1 % a.KU != 0;
    auto seg_range = [&](int k, int &us, int &ue) {
        const int t = seg_t0 + (seg_rot ? (k == 0 ? seg_n - 1 : k - 1) : k);
        us = max(u0, t * a.KU);
        ue = min(u1, (t + 1) * a.KU);
    };
    // The first two segments (the second empty if there is none).
    int pre_s0, pre_e0, pre_s1 = 0, pre_e1 = 0;
    seg_range(0, pre_s0, pre_e0);
    if (seg_n > 1)
        seg_range(1, pre_s1, pre_e1);

    if (warp == 0) {
        // ---------------------------------------------- codes + scales TMA --
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            const uint64_t pol_x = policy_evict_normal();
            int n = 0;
            bool go = true;
            for (int k = 0; k < seg_n && go; k++) {
              int us, ue;
              seg_range(k, us, ue);
              for (int u = us; u < ue; u++, n++) {
                // after the first unit, let the first segments' scale reads
                // land before the weight stream takes the memory system
                if (aborted() || (n == 1 && !wait(bar_pre, 0))) {
                    go = false;
                    break;
                }
                const int slot = n % CS;
                if (!wait(bar_cempty[slot], ((n / CS) & 1) ^ 1)) {
                    go = false;
                    break;
                }
                const int tile = u / a.KU, ku = u % a.KU;
                const uint32_t bar = smem_u32(&bar_cfull[slot]);
                const uint32_t dst = ring_s + slot * SLOT;
                mbar_arrive_expect_tx(bar, SLOT);
                if constexpr (FMT == 4) {
                    tma_load_2d(dst, &a.tm_codes, bar, ku * 128, tile * TM, pol);
                } else {
                    tma_load_2d(dst, &a.tm_codes, bar, ku * 256, tile * TM, pol);
                    tma_load_2d(dst + TM * 128, &a.tm_codes, bar, ku * 256 + 128, tile * TM, pol);
                }
#pragma unroll
                for (int j = 0; j < 4; j++)     // x: the unit's four 64-wide sub-tiles (L2-resident)
                    tma_load_2d(dst + CB + j * XB, &a.tm_x, bar, ku * kUnitK + j * kXK, 0, pol_x);
                tma_load_2d(dst + CB + 4 * XB, &a.tm_scales, bar, ku * 8, tile * TM, pol);
              }
            }
            // Drain: every load issued lands before the CTA may exit.
            for (int j = max(0, n - CS); j < n; j++)
                (void)mbar_wait_bounded(smem_u32(&bar_cfull[j % CS]), (j / CS) & 1);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA ----
        if (lane == 0) {
            constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(NB >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
            int i = 0, nu = 0;
            bool ok = true;
            for (int seg = 0; seg < seg_n && ok; seg++) {
                int us, uend;
                seg_range(seg, us, uend);
                const int buf = seg & 1;
                if (!wait(bar_accempty[buf], ((seg >> 1) & 1) ^ 1))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * 32);
                bool first = true;
                for (int u = us; u < uend && ok; u++, nu++) {
                    const int ns = nsub(u);
                    const int cslot = nu % CS;
                    // One wait a unit: every dequant warp has stored the unit's A
                    // (all its sub-stages).  They arrive only after seeing the
                    // unit's loads land, so x is in place too.  (A wait in this
                    // thread stalls the tensor pipe for its whole latency: the
                    // MMA queue is short.)  The dequant runs at most AS
                    // sub-stages, so at most AS units, ahead: AS barriers.
                    if (!wait(bar_ufull[nu % AS], (nu / AS) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < ns; j++, i++) {
                        const int slot = i % AS;
                        const uint32_t at = tmem + (uint32_t)(kAccCols + slot * kACols);
#pragma unroll
                        for (int kk = 0; kk < kSubK / 16; kk++) {
                            // K step of 16: 8 TMEM columns of A; x tile 2 j + kk / 4, 32
                            // bytes a step along its swizzled rows
                            const uint64_t bd = desc_k_sw128(ring_s + cslot * SLOT + CB + (2 * j + kk / 4) * XB);
                            umma_f16_ts(d_tmem, at + (uint32_t)(8 * kk), bd + (uint64_t)(2 * (kk % 4)), idesc,
                                        (first && kk == 0) ? 0u : 1u);
                        }
                        first = false;
                        umma_commit(smem_u32(&bar_aempty[slot]));
                    }
                    if (ok)     // the unit's x is read once these MMAs complete
                        umma_commit(smem_u32(&bar_cempty[cslot]));
                }
                if (!ok)
                    break;
                umma_commit(smem_u32(&bar_accfull[buf]));
            }
            // Every MMA issued has completed before TMEM is freed.
            umma_commit(smem_u32(&bar_done));
            (void)mbar_wait_bounded(smem_u32(&bar_done), 0);
        }
    } else if (warp == 2 || warp == 3) {
        // --------------------------------------------------- row shifts ----
        // Each segment's row shifts, up to kShiftRing segments ahead of the
        // dequantisation.  The first two segments' shifts are computed by the
        // dequantisation warps at the start (they have nothing else to do
        // then; one row and segment a thread); warps 2-3 publish them, then
        // compute the later segments' (thread t: rows t and t + 64).
        const int t = threadIdx.x - 64;
        bool ok = wait(bar_pre, 0);
        if (ok && lane == 0) {
            mbar_arrive(smem_u32(&bar_shift[0]));
            if (seg_n > 1)
                mbar_arrive(smem_u32(&bar_shift[1]));
        }
        for (int seg = 2; seg < seg_n && ok; seg++) {
            int u, uend;
            seg_range(seg, u, uend);
            const int tile = u / a.KU;
            const unsigned m0 = row_scale_max(tile, u, uend - u, t);
            const unsigned m1 = row_scale_max(tile, u, uend - u, t + 64);
            // (the slot's segment seg - kShiftRing must have been read)
            if (!wait(bar_shift_free[seg % kShiftRing], ((seg / kShiftRing) & 1) ^ 1))
                break;
            shift_s[seg % kShiftRing][t] = shift_of(m0);
            shift_s[seg % kShiftRing][t + 64] = shift_of(m1);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bar_shift[seg % kShiftRing]));
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        // ----------------------------------------------------- epilogue ----
        // (Warp w reads TMEM lanes 32 (w % 4) .. + 31: warps 4-7 cover all.)
        // Every cross-warp step here is an mbarrier with a bounded wait, so a
        // role that gave up on a timeout cannot leave the others blocked.
        const int q = warp - kEpiWarp0;          // TMEM lanes 32q .. 32q + 31
        const int r = 32 * q + lane;             // row within the tile
        int nsplit = 0, nepa = 0, nepb = 0;   // split tiles; phases of the handshake barriers
        for (int seg = 0; seg < seg_n; seg++) {
            int us, ue;
            seg_range(seg, us, ue);
            const int tile = us / a.KU;
            const int buf = seg & 1;
            if (!wait(bar_shift[seg % kShiftRing], (seg / kShiftRing) & 1))
                break;
            const int sh = shift_s[seg % kShiftRing][r];
            __syncwarp();
            if (lane == 0)                                 // the slot may take a later segment's shifts
                mbar_arrive(smem_u32(&bar_shift_free[seg % kShiftRing]));
            if (!__all_sync(0xffffffffu, wait(bar_accfull[buf], (seg >> 1) & 1)))
                break;                                     // (warp-uniform: tmem_ld is warp-collective)
            tc_fence_after();
            float v[NB];
            tmem_ld<NB>(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * 32), v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bar_accempty[buf]));
            // undo the row's power-of-two prescale (exact)
            const float unsc = __int_as_float((127 - sh) << 23);
#pragma unroll
            for (int b = 0; b < NB; b++)
                v[b] *= unsc;
            const int row = tile * TM + r;
            const long long tu0 = (long long)tile * a.KU;
            const int cf = owner_of(tu0, a.U, a.G), cl = owner_of(tu0 + a.KU - 1, a.U, a.G);
            if (cf == cl) {
                if (row < a.N) {
#pragma unroll
                    for (int b = 0; b < NB; b++)
                        if (b < a.B)
                            a.y[(size_t)b * a.N + row] = v[b];
                }
                continue;
            }
            // Tile split across CTAs (cf .. cl).  Whichever CTA completes the
            // tile last adds every part in CTA order (its own from registers),
            // so the sum does not depend on which CTA that is.  It usually
            // knows at once: the CTA holding the tile's first units reaches
            // them at the end of its range, after the others (which did theirs
            // at the start of theirs) have published.  So first an acquire
            // load of the tile's arrival count; only if some part is still
            // missing does this CTA publish its partial (slot 0: the tile of
            // its first unit, 1: of its last) and count its arrival, the
            // arrival that completes the count doing the sum.
            // Handshake (all bounded mbarriers): epi_b (1 arrival: thread 0
            // has put a count in epi_old) and epi_a (128: every thread is done
            // with epi_old, or has stored its partial).  Thread 0 writes
            // epi_old only after an epi_a phase, so neither barrier gets more
            // than one phase ahead of a waiter.
            const int others = cl - cf;
            if (r == 0) {
                if (nsplit > 0 && !wait(bar_epi_a, nepa++ & 1))
                    break;
                epi_old = ld_acquire_gpu_int(a.counters + tile);
                mbar_arrive(smem_u32(&bar_epi_b));
            }
            if (!wait(bar_epi_b, nepb++ & 1))
                break;
            int seen = epi_old;
            nsplit++;
            bool published = false;
            const int my_slot = (tile == u0 / a.KU) ? 0 : 1;
            if (seen != others) {
                float4 *dst = reinterpret_cast<float4 *>(a.partials + (((size_t)cta * 2 + my_slot) * TM + r) * 32);
#pragma unroll
                for (int b4 = 0; b4 < NB / 4; b4++)
                    __stcg(dst + b4, make_float4(v[4 * b4], v[4 * b4 + 1], v[4 * b4 + 2], v[4 * b4 + 3]));
                __threadfence();
                mbar_arrive(smem_u32(&bar_epi_a));
                if (r == 0) {
                    if (!wait(bar_epi_a, nepa++ & 1))
                        break;
                    epi_old = atom_add_acq_rel_gpu(a.counters + tile, 1);
                    mbar_arrive(smem_u32(&bar_epi_b));
                }
                if (!wait(bar_epi_b, nepb++ & 1))
                    break;
                seen = epi_old;
                published = true;
            }
            mbar_arrive(smem_u32(&bar_epi_a));      // done with epi_old
            if (seen != others)
                continue;
            float t[NB];
#pragma unroll
            for (int b = 0; b < NB; b++)
                t[b] = 0.f;
            for (int c = cf; c <= cl; c++) {
                const int cu0 = (int)((long long)c * a.U / a.G);
                const int sl = (tile == cu0 / a.KU) ? 0 : 1;
                float4 *src = reinterpret_cast<float4 *>(a.partials + (((size_t)c * 2 + sl) * TM + r) * 32);
                if (c == cta) {
#pragma unroll
                    for (int b = 0; b < NB; b++)
                        t[b] += v[b];
                    if (published) {
#pragma unroll
                        for (int b4 = 0; b4 < NB / 4; b4++)
                            __stcg(src + b4, make_float4(0.f, 0.f, 0.f, 0.f));
                    }
                    continue;
                }
                float4 pv[NB / 4];
#pragma unroll
                for (int b4 = 0; b4 < NB / 4; b4++)
                    pv[b4] = __ldcg(src + b4);
                // cleared once read: the workspace is all-zero again when the
                // call ends, so calls of any shape may share it
#pragma unroll
                for (int b4 = 0; b4 < NB / 4; b4++) {
                    __stcg(src + b4, make_float4(0.f, 0.f, 0.f, 0.f));
                    t[4 * b4] += pv[b4].x;
                    t[4 * b4 + 1] += pv[b4].y;
                    t[4 * b4 + 2] += pv[b4].z;
                    t[4 * b4 + 3] += pv[b4].w;
                }
            }
            if (row < a.N) {
#pragma unroll
                for (int b = 0; b < NB; b++)
                    if (b < a.B)
                        a.y[(size_t)b * a.N + row] = t[b];
            }
            if (r == 0)
                a.counters[tile] = 0;
        }
    } else if (warp >= kDequantWarp0) {
        // ------------------------------------------------ dequantisation ----
        // Warp w writes TMEM lanes 32 (w % 4) .. + 31, so warp w serves rows
        // r = 32 (w % 4) + lane, block h = (w - 8) / 4 of each 64-weight
        // sub-stage: a thread turns its (row, block) into 32 fp16 weights and
        // stores them as 16 TMEM columns of its lane.
        const int q = warp & 3, h = ((warp - kDequantWarp0) >> 2) & 1;
        const int grp = (warp - kDequantWarp0) >> 3;       // takes the sub-stages i with i % kDqGroups == grp
        const int r = 32 * q + lane;                       // row within the tile
        const int rsw = r & 7;                             // the 128-byte swizzle's XOR
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        {
            // the first two segments' row shifts: thread (j, row) of 256
            const int tid = threadIdx.x - 32 * kDequantWarp0;
            const int j = tid >> 7, rr = tid & (TM - 1);
            if (tid < 2 * TM && (j == 0 || seg_n > 1))
                shift_s[j][rr] = shift_of(j == 0 ? row_scale_max(pre_s0 / a.KU, pre_s0, pre_e0 - pre_s0, rr)
                                                 : row_scale_max(pre_s1 / a.KU, pre_s1, pre_e1 - pre_s1, rr));
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bar_pre));
        }
        int i = 0, n = 0;
        bool ok = true;
        for (int seg = 0; seg < seg_n && ok; seg++) {
            int u, uend;
            seg_range(seg, u, uend);
            // This segment's row shift (warps 2-3 computed it ahead).
            if (!wait(bar_shift[seg % kShiftRing], (seg / kShiftRing) & 1))
                break;
            const int s = shift_s[seg % kShiftRing][r];
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bar_shift_free[seg % kShiftRing]));
            const float two_s = __int_as_float((127 + s) << 23);
            for (; u < uend && ok; u++, n++) {
                const int cslot = n % CS;
                if (!__all_sync(0xffffffffu, wait(bar_cfull[cslot], (n / CS) & 1))) {
                    ok = false;
                    break;
                }
                const uint32_t crow = ring_s + cslot * SLOT + r * 128;
                const uint32_t srow_s = ring_s + cslot * SLOT + CB + 4 * XB + r * 16;
                const int ns = nsub(u);
                for (int j = 0; j < ns; j++, i++) {
                    if (i % kDqGroups != grp)
                        continue;
                    const int slot = i % AS;
                    // (warp-uniform outcome: the TMEM stores and their wait are
                    // warp-collective)
                    if (!__all_sync(0xffffffffu, wait(bar_aempty[slot], ((i / AS) & 1) ^ 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // this thread's two blocks of the sub-stage: 4 j + 2 h and
                    // 4 j + 2 h + 1 (64 consecutive weights, 32 TMEM columns)
                    uint32_t o[32];
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int blk = 4 * j + 2 * h + e;               // block of the unit (0..7)
                        unsigned short dbits;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(dbits) : "r"(srow_s + 2 * blk));
                        const float ds = __half2float(__ushort_as_half(dbits)) * two_s;
                        const __half2 ds2h = __float2half2_rn(ds);
                        uint32_t ds2;
                        memcpy(&ds2, &ds2h, 4);
                        uint32_t (&oe)[16] = *reinterpret_cast<uint32_t (*)[16]>(o + 16 * e);
                        if constexpr (FMT == 4) {
                            const uint4 c = lds128_u32(crow + ((blk ^ rsw) << 4));
                            dequant_q4_block(c, ds2, oe);
                        } else {
                            const uint32_t box = crow + (blk >> 2) * (TM * 128);
                            const int g = 2 * (blk & 3);
                            const uint4 c0 = lds128_u32(box + ((g ^ rsw) << 4));
                            const uint4 c1 = lds128_u32(box + (((g + 1) ^ rsw) << 4));
                            dequant_q8_half(c0, ds2, oe);
                            dequant_q8_half(c1, ds2, oe + 8);
                        }
                    }
                    tmem_st32(lane_base + (uint32_t)(kAccCols + slot * kACols + 32 * h), o);
                }
                // one wait for the unit's stores (they overlap the next
                // sub-stage's dequantisation; also on the way out, so none is
                // in flight when the columns are freed), then the hand-off
                tmem_wait_st();
                if (!ok)
                    break;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&bar_ufull[n % AS]));
                    mbar_arrive(smem_u32(&bar_cempty[cslot]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemCols);
}

}  // namespace vg

namespace {

template <int FMT, int NB>
int32_t verify_prepare()
{
    static std::atomic<bool> done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire))
        return BQ_OK;
    if (cudaFuncSetAttribute((const void *)vg::verify_gemm_kernel<FMT, NB>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)vg::smem_bytes<FMT, NB>()) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64)
        done[dev].store(true, std::memory_order_release);
    return BQ_OK;
}

struct VGeometry {
    int ntiles, KU, U, G;
};

VGeometry verify_geometry(long long N, long long K, int sms)
{
    VGeometry g;
    g.ntiles = (int)((N + vg::TM - 1) / vg::TM);
    g.KU = (int)((K + vg::kUnitK - 1) / vg::kUnitK);
    g.U = g.ntiles * g.KU;
    g.G = std::min(std::min(sms, vg::kMaxCtas), g.U);
    return g;
}

template <int FMT, int NB>
int32_t verify_launch(const bq_qmat *W, const uint16_t *x, int32_t B, float *y, void *ws,
                      int32_t *dev_status, void *stream, const VGeometry &geo)
{
    int32_t st = verify_prepare<FMT, NB>();
    if (st != BQ_OK)
        return st;
    vg::Args a;
    memset(&a, 0, sizeof(a));
    const int N = W->N, K = W->K;
    const uint64_t cdims[2] = {(uint64_t)(FMT == 4 ? K / 2 : K), (uint64_t)N};
    const uint64_t cstr[1] = {(uint64_t)(FMT == 4 ? K / 2 : K)};
    const uint32_t cbox[2] = {128u, (uint32_t)vg::TM};
    const int ldS = bq_scales_ld(K);
    const uint64_t sdims[2] = {(uint64_t)(K / 32), (uint64_t)N};
    const uint64_t sstr[1] = {(uint64_t)ldS * 2};
    const uint32_t sbox[2] = {8u, (uint32_t)vg::TM};
    const uint64_t xdims[2] = {(uint64_t)K, (uint64_t)B};
    const uint64_t xstr[1] = {(uint64_t)K * 2};
    const uint32_t xbox[2] = {(uint32_t)vg::kXK, (uint32_t)NB};
    if (!encode_tensor_map(&a.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, W->codes, cdims, cstr, cbox,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !encode_tensor_map(&a.tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W->scales, sdims, sstr,
                           sbox, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE) ||
        !encode_tensor_map(&a.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x, xdims, xstr, xbox,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
        return BQ_ERR_CUDA;
    a.scales = W->scales;
    a.y = y;
    a.N = N;
    a.K = K;
    a.B = B;
    a.ldS = ldS;
    a.ntiles = geo.ntiles;
    a.KU = geo.KU;
    a.U = geo.U;
    a.G = geo.G;
    a.counters = static_cast<int *>(ws);
    a.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                           align_up((size_t)geo.ntiles * sizeof(int), 256));
    a.status = dev_status;
    void *args[] = {&a};
    cudaError_t e = launch_pdl((const void *)vg::verify_gemm_kernel<FMT, NB>, dim3(geo.G),
                               dim3(vg::kThreads), vg::smem_bytes<FMT, NB>(),
                               static_cast<cudaStream_t>(stream), args);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_verify_workspace_bytes(int32_t N, int32_t K, int32_t B)
{
    if (N < 1 || K < 32 || K % 32 != 0 || B < 1 || B > 32)
        return 0;
    const long long ntiles = ((long long)N + vg::TM - 1) / vg::TM;
    return align_up((size_t)ntiles * sizeof(int), 256) + (size_t)vg::kMaxCtas * vg::kPartBytesPerCta;
}

extern "C" int32_t bq_verify_gemm(int32_t fmt, const bq_qmat *W, const uint16_t *x, int32_t B,
                                  float *y, void *ws, size_t ws_bytes, int32_t *dev_status,
                                  void *stream)
{
    int32_t st = check_qmat(W);
    if (st != BQ_OK)
        return st;
    if (fmt != 4 && fmt != 8)
        return BQ_ERR_SHAPE;
    if (!x || !y || !ws)
        return BQ_ERR_NULL;
    if (B < 1 || B > 32)
        return BQ_ERR_BATCH;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws))
        return BQ_ERR_ALIGN;
    if (ws_bytes < bq_verify_workspace_bytes(W->N, W->K, B))
        return BQ_ERR_WORKSPACE;
    const int sms = device_sm_count();
    if (sms <= 0)
        return BQ_ERR_CUDA;
    const VGeometry geo = verify_geometry(W->N, W->K, sms);
    if ((long long)geo.ntiles * geo.KU >= (1LL << 31) / 2)
        return BQ_ERR_SHAPE;
    if (fmt == 4)
        return B <= 16 ? verify_launch<4, 16>(W, x, B, y, ws, dev_status, stream, geo)
                       : verify_launch<4, 32>(W, x, B, y, ws, dev_status, stream, geo);
    return B <= 16 ? verify_launch<8, 16>(W, x, B, y, ws, dev_status, stream, geo)
                   : verify_launch<8, 32>(W, x, B, y, ws, dev_status, stream, geo);
}
