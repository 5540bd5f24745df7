// bq_device.cuh -- device building blocks of the streamed block-quantised GEMV
// for sm_100a: PTX wrappers (mbarrier, TMA tensor loads, mma.sync,
// programmatic dependent launch), in-register dequantisation of every format
// and the per-chunk dot product.
//
// Work unit ("chunk"): kRows weight rows (32 or 16 for Q4, 16 for the other
// formats) x 256 weights along K (8 blocks of 32).  A Q4 / Q8 chunk's codes
// arrive in shared memory through one (Q4: kRows x 128 bytes) or two (Q8: 16
// rows x 128 bytes each) 2-D TMA boxes with the 128-byte swizzle (the other
// formats: see their traits below), its scales through one kRows x 8 fp16
// box.  A warp reads them with 32-bit shared loads that the swizzle makes
// bank-conflict free, turns each 4-byte group into fp16 pairs in registers
// (exact: see "dequant" below), and forms the block's partial dot products
// with m16n8k16 mma.sync (fp16 in, fp32 accumulate): M = 16 weight rows (a
// 32-row Q4 chunk is two such m-tiles that share every x fragment), N = the
// batch (B <= 8), K = 16 elements of one block.  Each block's partial sum is
// scaled by its fp32-converted scale once (y += d * sum((q - z) x)), so the
// only roundings are fp32 ones.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <string.h>

#ifndef BQ_WARPS
#define BQ_WARPS 8          // worker warps per CTA
#endif

namespace bq {

constexpr int kBlock = 32;          // weights per quantisation block
constexpr int kChunkK = 256;        // weights along K per chunk
constexpr int kWarps = BQ_WARPS;    // worker warps per CTA
constexpr int kMaxCluster = 8;      // CTAs of a cluster (portable limit)
constexpr int kThreads = kWarps * 32;

// Status bits OR-ed into the caller's device status word (1 << bq_status).
constexpr int kStatusExpertIndex = 1 << 5;
constexpr int kStatusTimeout = 1 << 7;
constexpr int kStatusRange = 1 << 9;

// A bounded wait gives up after this many SM clock cycles (~2 s).
constexpr long long kWaitCycles = 4000000000LL;

// Tuning knobs (compile-time; the defaults are the measured best on B200).
#ifndef BQ_Q4_MT
#define BQ_Q4_MT 2          // 16-row m-tiles per Q4 chunk where no geometry is chosen per call
#endif
#ifndef BQ_CLUSTER_SUMS
#define BQ_CLUSTER_SUMS 1   // matrix mode: cross-CTA band sums through a cluster's shared memory
#endif
#ifndef BQ_STAGES
#define BQ_STAGES 2         // ring slots per worker warp
#endif
#ifndef BQ_MIN_BLOCKS
#define BQ_MIN_BLOCKS 2     // CTAs per SM the register budget is sized for
#endif

// Chunk geometry of a format: MT m-tiles of 16 rows.  Q4 comes in two: 32-row
// chunks (MT = 2, two m-tiles share every x fragment: fewer instructions per
// weight) and 16-row chunks (MT = 1: twice the work units, for launches too
// small to give every warp a 32-row chunk).  Q8, Q2, Q3, Q5 and Q6 chunks are 16 rows.
template <int FMT>
__host__ __device__ constexpr int default_mt()
{
    return FMT == 4 ? BQ_Q4_MT : 1;
}
// Q6 chunks: 16 rows x 256 weights, the low-nibble plane as one 128-byte box
// (Q4's layout, 128-byte swizzle) and the top-bit plane as one 64-byte box
// after it (no swizzle): 3 KB of codes per chunk.
template <int FMT, int MT = default_mt<FMT>()> struct Fmt;
template <int MT> struct Fmt<4, MT> {
    static_assert(MT == 1 || MT == 2, "Q4 chunks are 16 or 32 rows");
    static constexpr int kMT = MT;                      // m-tiles of 16 rows per chunk
    static constexpr int kRows = 16 * kMT;              // rows per chunk / band
    static constexpr int kBoxes = 1;                    // code boxes of the first plane
    static constexpr int kLoRow = 128;                  // bytes per row of one such box
    static constexpr int kCodeBytes = kRows * 128;      // 2 or 4 KB
    static constexpr int kCodeLoad = kCodeBytes;        // code bytes one chunk's loads bring
    static constexpr int kScaleBytes = kRows * 16;      // kRows x 8 fp16
    static constexpr int kStages = BQ_STAGES;
};
// Q5 likewise, with a 32-byte top-bit box: 2.5 KB of codes per chunk, in a
// 3 KB slot (slots stay 1024-byte aligned, as the 128-byte swizzle of the
// low-nibble box assumes).
template <int FMT> struct FmtTop {
    static constexpr int kMT = 1;
    static constexpr int kRows = 16;
    static constexpr int kBoxes = 1;                    // + the top-bit box
    static constexpr int kLoRow = 128;
    static constexpr int kTopRow = FMT == 6 ? 64 : 32;  // top-bit bytes per row and chunk
    static constexpr int kCodeLoad = kRows * 128 + kRows * kTopRow;
    static constexpr int kCodeBytes = 3072;             // slot stride
    static constexpr int kScaleBytes = kRows * 16;
    static constexpr int kStages = BQ_STAGES;
};
template <> struct Fmt<6, 1> : FmtTop<6> {};
template <> struct Fmt<5, 1> : FmtTop<5> {};
// Q2 / Q3 chunks: 16 rows x 256 weights, the 2-bit plane as one 64-byte box
// (64-byte swizzle: slots 512-byte aligned) and, for Q3, the 1-bit plane as
// one 32-byte box after it (no swizzle): 1 KB / 1.5 KB of codes per chunk.
template <int FMT> struct FmtLow2 {
    static constexpr int kMT = 1;
    static constexpr int kRows = 16;
    static constexpr int kBoxes = 1;                    // (+ the top-bit box for Q3)
    static constexpr int kLoRow = 64;
    static constexpr int kTopRow = FMT == 3 ? 32 : 0;
    static constexpr int kCodeLoad = kRows * (kLoRow + kTopRow);
    static constexpr int kCodeBytes = kCodeLoad;        // slot stride: 1024 or 1536
    static constexpr int kScaleBytes = kRows * 16;
    static constexpr int kStages = BQ_STAGES;
};
template <> struct Fmt<2, 1> : FmtLow2<2> {};
template <> struct Fmt<3, 1> : FmtLow2<3> {};
template <> struct Fmt<8, 1> {
    static constexpr int kMT = 1;
    static constexpr int kRows = 16;
    static constexpr int kBoxes = 2;
    static constexpr int kLoRow = 128;
    static constexpr int kCodeBytes = 2 * kRows * 128;  // 4 KB
    static constexpr int kCodeLoad = kCodeBytes;
    static constexpr int kScaleBytes = kRows * 16;
    static constexpr int kStages = BQ_STAGES;
};
static_assert(Fmt<5, 1>::kCodeLoad <= Fmt<5, 1>::kCodeBytes &&
                  Fmt<6, 1>::kCodeLoad <= Fmt<6, 1>::kCodeBytes && Fmt<4, 2>::kCodeBytes % 1024 == 0 &&
                  Fmt<5, 1>::kCodeBytes % 1024 == 0 && Fmt<6, 1>::kCodeBytes % 1024 == 0 &&
                  Fmt<8, 1>::kCodeBytes % 1024 == 0,
              "code slots hold a chunk and stay 1024-byte aligned");
static_assert(Fmt<2, 1>::kCodeBytes % 512 == 0 && Fmt<3, 1>::kCodeBytes % 512 == 0,
              "Q2 / Q3 code slots stay 512-byte aligned (the 64-byte swizzle's period)");

template <int FMT, int MT = default_mt<FMT>()>
constexpr int smem_bytes()
{
    using F = Fmt<FMT, MT>;
    return kWarps * F::kStages * (F::kCodeBytes + F::kScaleBytes) + kWarps * F::kStages * 8 + 1024;
}

// ------------------------------------------------------------------ PTX ----
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// The same wait with cluster-scope acquire: for data other CTAs of the
// cluster stored into this CTA's shared memory (st_async_v4).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Pass a value through an opaque volatile asm: anything computed from the
// result is ordered after every earlier volatile asm (e.g. an mbarrier wait),
// even when it is itself a non-volatile asm with no memory clobber.
__device__ __forceinline__ uint32_t launder(uint32_t v)
{
    uint32_t r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v) : "memory");
    return r;
}

// Non-blocking test of phase `parity` of an mbarrier.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

#ifndef BQ_WAIT_TEST_FIRST
#define BQ_WAIT_TEST_FIRST 1
#endif

// Wait for phase `parity` of an mbarrier, giving up after kWaitCycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
#if BQ_WAIT_TEST_FIRST
    if (mbar_test_wait(bar, parity))
        return true;
#endif
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitCycles)
            return false;
    }
    return true;
}

__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (clock64() - t0 > kWaitCycles)
            return false;
    }
    return true;
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}

// ------------------------------------------------------------ clusters ----
__device__ __forceinline__ uint32_t cluster_nctarank()
{
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}
// Every thread of every CTA of the cluster arrives (release) and waits
// (acquire): shared-memory state set up before it is visible cluster-wide.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
__device__ __forceinline__ void fence_mbarrier_init_cluster()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// The shared::cluster address of `addr` (a shared::cta address) in the CTA
// of cluster rank `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// 16 bytes into another CTA's shared memory; completes 16 bytes of that
// CTA's mbarrier transaction count.
__device__ __forceinline__ void st_async_v4(uint32_t remote, float4 v, uint32_t remote_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 ::"r"(remote), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(remote_bar) : "memory");
}

// Pull the 128-byte line holding p into L1.
__device__ __forceinline__ void prefetch_l1(const void *p)
{
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch: let the next kernel on the stream be
// scheduled, and wait until the previous one has completed and its writes are
// visible.  Both are no-ops when the launch carries no PDL attribute.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 8 bytes of x.  COHERENT = false: the read-only path, kept in L1 (every warp
// of the SM re-reads the same activations for every band) -- valid when
// nothing in the launch writes x.  COHERENT = true: an ordinary (weak) load,
// L1-cached, for x that an earlier stage of the same launch may have written:
// it is issued after the grid barrier's GPU-scope acquire, which the memory
// model requires to make those writes visible to it (no stale L1 line).
template <bool COHERENT>
__device__ __forceinline__ uint2 ldg64(const void *p)
{
    uint2 v;
    if constexpr (COHERENT)
        asm volatile("ld.global.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
    else
        asm("ld.global.nc.L1::evict_last.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Release / acquire read-modify-writes at GPU scope (no separate fence).
__device__ __forceinline__ int atom_add_release_gpu(int *p, int v)
{
    int old;
    asm volatile("atom.add.release.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v)
{
    int old;
    asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// D = A(16x16 f16) * B(16x8 f16) + C, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1, const float (&c)[4])
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// ------------------------------------------------------------- dequant ----
// The mma fragment of a block half: lane (g = lane/4, t = lane%4) supplies
// for its rows g and g+8 the k-slots {2t, 2t+1} and {2t+8, 2t+9}.  We map
// slot pair {2t, 2t+1} -> elements {4t, 4t+1} and {2t+8, 2t+9} -> {4t+2, 4t+3}
// of the half (a bijection of the 16 slots), so a lane's four elements are
// the 4 consecutive code bytes 4t..4t+3 it loads, and its x fragment is the
// 4 consecutive x values at the same k -- one 8-byte load, no shuffles.
//
// Codes enter the tensor core as fp16 *subnormals*: a 16-bit lane holding the
// integer u (< 1024) in its low bits and zero elsewhere is exactly u * 2^-24,
// so masking the code bits into place is the whole conversion.  Q8: the byte
// biased by +128 (u = q + 128).  Q4: both nibbles of a byte are placed at bits
// 4-7 of their lanes (u = 16 q): the high nibble is already there, the low one
// gets there by a multiply by 16 -- on the FMA pipe, which leaves the ALU pipe
// (the busier one) one operation per register instead of two.  Either way the
// lane is z' + u for a zero point z' = 128 (8 * 16 for Q4), removed by a second
// mma that starts each block's accumulator at -128 * 2^-24 * sum(x)
// (block_offset).  Every product is exact; the scale 2^-24 (2^-20 for Q4) is
// undone at the store.

// f16x2 of -z' * 2^-24: z' = 128 (Q4: 8 * 16; Q8: 128), 256 (Q5: 16 * 16),
// 512 (Q6: 32 * 16; Q2: 2 * 256) or 1024 (Q3: 4 * 256, the smallest normal).
template <int FMT>
__host__ __device__ constexpr uint32_t zero_point_pair()
{
    return FMT == 3 ? 0x84008400u
                    : (FMT == 6 || FMT == 2 ? 0x82008200u : (FMT == 5 ? 0x81008100u : 0x80808080u));
}

// The y of a band is stored as acc * 2^20 (Q4, Q5, Q6: codes enter at
// 16 * 2^-24), acc * 2^16 (Q2, Q3: at 256 * 2^-24) or acc * 2^24 (Q8).
template <int FMT>
__host__ __device__ constexpr float unscale()
{
    return FMT == 8 ? 16777216.0f : (FMT == 2 || FMT == 3 ? 65536.0f : 1048576.0f);
}

__device__ __forceinline__ float half_lo(uint32_t v)
{
    __half2 h;
    memcpy(&h, &v, 4);
    return __low2float(h);
}
__device__ __forceinline__ float half_hi(uint32_t v)
{
    __half2 h;
    memcpy(&h, &v, 4);
    return __high2float(h);
}
__device__ __forceinline__ uint32_t pick_u32(const uint4 &v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// sum(x) of one block, pre-multiplied by -z * 2^-24, in the accumulator
// layout (rows are all equal): the starting value of the block's mma chain.
template <int FMT>
__device__ __forceinline__ void block_offset(uint2 xa, uint2 xb, float (&s)[4])
{
    const uint32_t z = zero_point_pair<FMT>();
    asm("{\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%4,%4,%4}, {%5,%6}, "
        "{%9,%9,%9,%9};\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%4,%4,%4}, {%7,%8}, "
        "{%0,%1,%2,%3};\n\t}"
        : "=&f"(s[0]), "=&f"(s[1]), "=&f"(s[2]), "=&f"(s[3])
        : "r"(z), "r"(xa.x), "r"(xa.y), "r"(xb.x), "r"(xb.y), "f"(0.0f));
}

// One Q4 block (32 weights along K) for one 16-row m-tile, in PTX so the
// instruction sequence is exactly: 2 shared loads (rows g, g+8), 4 prmt to
// spread the 4 code bytes of each row over fp16 lanes, 4 multiplies by 16
// (`m16` holds 16 in a register, so they stay multiplies) and 8 masks to place
// each nibble at bits 4-7, 2 mma (low then high nibbles, starting from the
// zero-point term `off`), 4 fma for the scales.  `addr` is the shared address
// of row g's 4-byte group.
__device__ __forceinline__ void block_q4(uint32_t addr, uint2 xa, uint2 xb, const float (&off)[4],
                                         float dg, float dg8, float (&acc)[4], uint32_t m16)
{
    asm("{\n\t"
        ".reg .b32 w0, w8, p01, p23, q01, q23, a0, a1, a2, a3;\n\t"
        ".reg .f32 c0, c1, c2, c3;\n\t"
        "ld.shared.b32 w0, [%4];\n\t"
        "ld.shared.b32 w8, [%4+1024];\n\t"
        "prmt.b32 p01, w0, 0, 0x4140;\n\t"
        "prmt.b32 p23, w0, 0, 0x4342;\n\t"
        "prmt.b32 q01, w8, 0, 0x4140;\n\t"
        "prmt.b32 q23, w8, 0, 0x4342;\n\t"
        "mul.lo.u32 a0, p01, %15;\n\t"
        "mul.lo.u32 a1, q01, %15;\n\t"
        "mul.lo.u32 a2, p23, %15;\n\t"
        "mul.lo.u32 a3, q23, %15;\n\t"
        "and.b32 a0, a0, 0x00F000F0;\n\t"
        "and.b32 a1, a1, 0x00F000F0;\n\t"
        "and.b32 a2, a2, 0x00F000F0;\n\t"
        "and.b32 a3, a3, 0x00F000F0;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%5,%6}, "
        "{%9,%10,%11,%12};\n\t"
        "and.b32 a0, p01, 0x00F000F0;\n\t"
        "and.b32 a1, q01, 0x00F000F0;\n\t"
        "and.b32 a2, p23, 0x00F000F0;\n\t"
        "and.b32 a3, q23, 0x00F000F0;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%7,%8}, "
        "{c0,c1,c2,c3};\n\t"
        "fma.rn.f32 %0, %13, c0, %0;\n\t"
        "fma.rn.f32 %1, %13, c1, %1;\n\t"
        "fma.rn.f32 %2, %14, c2, %2;\n\t"
        "fma.rn.f32 %3, %14, c3, %3;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
        : "r"(addr), "r"(xa.x), "r"(xa.y), "r"(xb.x), "r"(xb.y), "f"(off[0]), "f"(off[1]),
          "f"(off[2]), "f"(off[3]), "f"(dg), "f"(dg8), "r"(m16));
}
// One Q6 or Q5 block for a 16-row m-tile: Q4's nibble placement (u = 16 *
// low 4 bits at bits 4-7) plus the top bits of each code at bits 8-9 (Q6: 2
// bits) or bit 8 (Q5: 1), so a lane holds u = 16 q exactly (q < 64, u <
// 1024).  `addr` is row g's 4-byte group of low nibbles (as block_q4);
// `addr_hi` row g's 4-byte group of top bits, whose byte i serves elements
// 4t+i and 4t+16+i: Q6 -- byte i of the group at 4(t%2) holds pairs of
// elements 4(t%2)+i+8p, pair t/2 for 4t+i and t/2+2 for 4t+16+i; Q5 -- byte
// i of the block's 4 bytes holds bits of elements i+4p, bit t for 4t+i and
// t+4 for 4t+16+i.  `mh1` / `mh2` (Q6: 2^(8-2(t/2)), 2^(4-2(t/2)); Q5:
// 2^(8-t), 2^(4-t)) move those bits to bit 8 (multiplies, on the FMA pipe).
// Row g+8 is 1024 bytes on in the low plane, 8 top rows on in the top plane.
template <int FMT>
__device__ __forceinline__ void block_qtop(uint32_t addr, uint32_t addr_hi, uint2 xa, uint2 xb,
                                           const float (&off)[4], float dg, float dg8,
                                           float (&acc)[4], uint32_t m16, uint32_t mh1,
                                           uint32_t mh2)
{
    constexpr uint32_t kTopMask = FMT == 6 ? 0x03000300u : 0x01000100u;
    constexpr int kTop8 = 8 * Fmt<FMT, 1>::kTopRow;   // row g+8 in the top plane
    asm("{\n\t"
        ".reg .b32 w0, w8, h0, h8, p01, p23, q01, q23, e01, e23, f01, f23, a0, a1, a2, a3, t0, t1, t2, t3;\n\t"
        ".reg .f32 c0, c1, c2, c3;\n\t"
        "ld.shared.b32 w0, [%4];\n\t"
        "ld.shared.b32 w8, [%4+1024];\n\t"
        "ld.shared.b32 h0, [%5];\n\t"
        "ld.shared.b32 h8, [%5+%19];\n\t"
        "prmt.b32 p01, w0, 0, 0x4140;\n\t"
        "prmt.b32 p23, w0, 0, 0x4342;\n\t"
        "prmt.b32 q01, w8, 0, 0x4140;\n\t"
        "prmt.b32 q23, w8, 0, 0x4342;\n\t"
        "prmt.b32 e01, h0, 0, 0x4140;\n\t"
        "prmt.b32 e23, h0, 0, 0x4342;\n\t"
        "prmt.b32 f01, h8, 0, 0x4140;\n\t"
        "prmt.b32 f23, h8, 0, 0x4342;\n\t"
        // elements 4t..4t+3: low nibble * 16 | top pair t/2 at bits 8-9
        "mul.lo.u32 a0, p01, %16;\n\t"
        "mul.lo.u32 a1, q01, %16;\n\t"
        "mul.lo.u32 a2, p23, %16;\n\t"
        "mul.lo.u32 a3, q23, %16;\n\t"
        "mul.lo.u32 t0, e01, %17;\n\t"
        "mul.lo.u32 t1, f01, %17;\n\t"
        "mul.lo.u32 t2, e23, %17;\n\t"
        "mul.lo.u32 t3, f23, %17;\n\t"
        "and.b32 t0, t0, %20;\n\t"
        "and.b32 t1, t1, %20;\n\t"
        "and.b32 t2, t2, %20;\n\t"
        "and.b32 t3, t3, %20;\n\t"
        "lop3.b32 a0, a0, 0x00F000F0, t0, 0xEA;\n\t"
        "lop3.b32 a1, a1, 0x00F000F0, t1, 0xEA;\n\t"
        "lop3.b32 a2, a2, 0x00F000F0, t2, 0xEA;\n\t"
        "lop3.b32 a3, a3, 0x00F000F0, t3, 0xEA;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%6,%7}, "
        "{%10,%11,%12,%13};\n\t"
        // elements 4t+16..4t+19: high nibble | top pair t/2 + 2 at bits 8-9
        "mul.lo.u32 t0, e01, %18;\n\t"
        "mul.lo.u32 t1, f01, %18;\n\t"
        "mul.lo.u32 t2, e23, %18;\n\t"
        "mul.lo.u32 t3, f23, %18;\n\t"
        "and.b32 t0, t0, %20;\n\t"
        "and.b32 t1, t1, %20;\n\t"
        "and.b32 t2, t2, %20;\n\t"
        "and.b32 t3, t3, %20;\n\t"
        "lop3.b32 a0, p01, 0x00F000F0, t0, 0xEA;\n\t"
        "lop3.b32 a1, q01, 0x00F000F0, t1, 0xEA;\n\t"
        "lop3.b32 a2, p23, 0x00F000F0, t2, 0xEA;\n\t"
        "lop3.b32 a3, q23, 0x00F000F0, t3, 0xEA;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%8,%9}, "
        "{c0,c1,c2,c3};\n\t"
        "fma.rn.f32 %0, %14, c0, %0;\n\t"
        "fma.rn.f32 %1, %14, c1, %1;\n\t"
        "fma.rn.f32 %2, %15, c2, %2;\n\t"
        "fma.rn.f32 %3, %15, c3, %3;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
        : "r"(addr), "r"(addr_hi), "r"(xa.x), "r"(xa.y), "r"(xb.x), "r"(xb.y), "f"(off[0]),
          "f"(off[1]), "f"(off[2]), "f"(off[3]), "f"(dg), "f"(dg8), "r"(m16), "r"(mh1), "r"(mh2),
          "n"(kTop8), "n"(kTopMask));
}

// One Q2 or Q3 block for a 16-row m-tile.  `addr` is row g's 4-byte group of
// the 2-bit plane at byte 4(t%2) of the block: its byte i holds elements
// 4(t%2)+i+8p in bit pair p, which puts element 4t+i in pair t/2 and element
// 4t+16+i in pair t/2+2.  After the bytes are spread over fp16 lanes, the
// multipliers mh1 = 2^(8-2(t/2)) and mh2 = 2^(4-2(t/2)) move those pairs to
// bits 8-9 (u = 256 * low 2 bits).  Q3 adds bit 2 of each code from
// `addr_hi`, row g's 4 bytes of the 1-bit plane (Q5's layout: bit t of byte
// i for element 4t+i, bit t+4 for 4t+16+i), moved to bit 10 by mh3 =
// 2^(10-t) and mh4 = 2^(6-t).  So a lane holds u = 256 q (q < 8, u < 2048):
// an fp16 subnormal, or from u = 1024 on a normal of the lowest binade,
// which is still exactly u * 2^-24.  Row g+8 is 8 rows on: 512 bytes in the
// 2-bit box, 256 in the 1-bit box.  The multiplies run on the FMA pipe.
template <int FMT>
__device__ __forceinline__ void block_q23(uint32_t addr, uint32_t addr_hi, uint2 xa, uint2 xb,
                                          const float (&off)[4], float dg, float dg8,
                                          float (&acc)[4], uint32_t mh1, uint32_t mh2,
                                          uint32_t mh3, uint32_t mh4)
{
    if constexpr (FMT == 2) {
        asm("{\n\t"
            ".reg .b32 w0, w8, p01, p23, q01, q23, a0, a1, a2, a3;\n\t"
            ".reg .f32 c0, c1, c2, c3;\n\t"
            "ld.shared.b32 w0, [%4];\n\t"
            "ld.shared.b32 w8, [%4+512];\n\t"
            "prmt.b32 p01, w0, 0, 0x4140;\n\t"
            "prmt.b32 p23, w0, 0, 0x4342;\n\t"
            "prmt.b32 q01, w8, 0, 0x4140;\n\t"
            "prmt.b32 q23, w8, 0, 0x4342;\n\t"
            "mul.lo.u32 a0, p01, %15;\n\t"
            "mul.lo.u32 a1, q01, %15;\n\t"
            "mul.lo.u32 a2, p23, %15;\n\t"
            "mul.lo.u32 a3, q23, %15;\n\t"
            "and.b32 a0, a0, 0x03000300;\n\t"
            "and.b32 a1, a1, 0x03000300;\n\t"
            "and.b32 a2, a2, 0x03000300;\n\t"
            "and.b32 a3, a3, 0x03000300;\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%5,%6}, "
            "{%9,%10,%11,%12};\n\t"
            "mul.lo.u32 a0, p01, %16;\n\t"
            "mul.lo.u32 a1, q01, %16;\n\t"
            "mul.lo.u32 a2, p23, %16;\n\t"
            "mul.lo.u32 a3, q23, %16;\n\t"
            "and.b32 a0, a0, 0x03000300;\n\t"
            "and.b32 a1, a1, 0x03000300;\n\t"
            "and.b32 a2, a2, 0x03000300;\n\t"
            "and.b32 a3, a3, 0x03000300;\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%7,%8}, "
            "{c0,c1,c2,c3};\n\t"
            "fma.rn.f32 %0, %13, c0, %0;\n\t"
            "fma.rn.f32 %1, %13, c1, %1;\n\t"
            "fma.rn.f32 %2, %14, c2, %2;\n\t"
            "fma.rn.f32 %3, %14, c3, %3;\n\t}"
            : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
            : "r"(addr), "r"(xa.x), "r"(xa.y), "r"(xb.x), "r"(xb.y), "f"(off[0]), "f"(off[1]),
              "f"(off[2]), "f"(off[3]), "f"(dg), "f"(dg8), "r"(mh1), "r"(mh2));
        (void)addr_hi;
        (void)mh3;
        (void)mh4;
    } else {
        asm("{\n\t"
            ".reg .b32 w0, w8, h0, h8, p01, p23, q01, q23, e01, e23, f01, f23, a0, a1, a2, a3, t0, t1, t2, t3;\n\t"
            ".reg .f32 c0, c1, c2, c3;\n\t"
            "ld.shared.b32 w0, [%4];\n\t"
            "ld.shared.b32 w8, [%4+512];\n\t"
            "ld.shared.b32 h0, [%5];\n\t"
            "ld.shared.b32 h8, [%5+256];\n\t"
            "prmt.b32 p01, w0, 0, 0x4140;\n\t"
            "prmt.b32 p23, w0, 0, 0x4342;\n\t"
            "prmt.b32 q01, w8, 0, 0x4140;\n\t"
            "prmt.b32 q23, w8, 0, 0x4342;\n\t"
            "prmt.b32 e01, h0, 0, 0x4140;\n\t"
            "prmt.b32 e23, h0, 0, 0x4342;\n\t"
            "prmt.b32 f01, h8, 0, 0x4140;\n\t"
            "prmt.b32 f23, h8, 0, 0x4342;\n\t"
            // elements 4t..4t+3: pair t/2 at bits 8-9 | bit t of the 1-bit group at bit 10
            "mul.lo.u32 a0, p01, %15;\n\t"
            "mul.lo.u32 a1, q01, %15;\n\t"
            "mul.lo.u32 a2, p23, %15;\n\t"
            "mul.lo.u32 a3, q23, %15;\n\t"
            "mul.lo.u32 t0, e01, %17;\n\t"
            "mul.lo.u32 t1, f01, %17;\n\t"
            "mul.lo.u32 t2, e23, %17;\n\t"
            "mul.lo.u32 t3, f23, %17;\n\t"
            "and.b32 t0, t0, 0x04000400;\n\t"
            "and.b32 t1, t1, 0x04000400;\n\t"
            "and.b32 t2, t2, 0x04000400;\n\t"
            "and.b32 t3, t3, 0x04000400;\n\t"
            "lop3.b32 a0, a0, 0x03000300, t0, 0xEA;\n\t"
            "lop3.b32 a1, a1, 0x03000300, t1, 0xEA;\n\t"
            "lop3.b32 a2, a2, 0x03000300, t2, 0xEA;\n\t"
            "lop3.b32 a3, a3, 0x03000300, t3, 0xEA;\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%6,%7}, "
            "{%10,%11,%12,%13};\n\t"
            // elements 4t+16..4t+19: pair t/2+2 | bit t+4
            "mul.lo.u32 a0, p01, %16;\n\t"
            "mul.lo.u32 a1, q01, %16;\n\t"
            "mul.lo.u32 a2, p23, %16;\n\t"
            "mul.lo.u32 a3, q23, %16;\n\t"
            "mul.lo.u32 t0, e01, %18;\n\t"
            "mul.lo.u32 t1, f01, %18;\n\t"
            "mul.lo.u32 t2, e23, %18;\n\t"
            "mul.lo.u32 t3, f23, %18;\n\t"
            "and.b32 t0, t0, 0x04000400;\n\t"
            "and.b32 t1, t1, 0x04000400;\n\t"
            "and.b32 t2, t2, 0x04000400;\n\t"
            "and.b32 t3, t3, 0x04000400;\n\t"
            "lop3.b32 a0, a0, 0x03000300, t0, 0xEA;\n\t"
            "lop3.b32 a1, a1, 0x03000300, t1, 0xEA;\n\t"
            "lop3.b32 a2, a2, 0x03000300, t2, 0xEA;\n\t"
            "lop3.b32 a3, a3, 0x03000300, t3, 0xEA;\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%8,%9}, "
            "{c0,c1,c2,c3};\n\t"
            "fma.rn.f32 %0, %14, c0, %0;\n\t"
            "fma.rn.f32 %1, %14, c1, %1;\n\t"
            "fma.rn.f32 %2, %19, c2, %2;\n\t"
            "fma.rn.f32 %3, %19, c3, %3;\n\t}"
            : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
            : "r"(addr), "r"(addr_hi), "r"(xa.x), "r"(xa.y), "r"(xb.x), "r"(xb.y), "f"(off[0]),
              "f"(off[1]), "f"(off[2]), "f"(off[3]), "f"(dg), "r"(mh1), "r"(mh2), "r"(mh3),
              "r"(mh4), "f"(dg8));
    }
}

// One Q8 block for the 16-row m-tile: addr_a / addr_b are row g's 4-byte
// groups in the block's two 16-element halves.
__device__ __forceinline__ void block_q8(uint32_t addr_a, uint32_t addr_b, uint2 xa, uint2 xb,
                                         const float (&off)[4], float dg, float dg8, float (&acc)[4])
{
    asm("{\n\t"
        ".reg .b32 w0, w8, v0, v8, a0, a1, a2, a3;\n\t"
        ".reg .f32 c0, c1, c2, c3;\n\t"
        "ld.shared.b32 w0, [%4];\n\t"
        "ld.shared.b32 w8, [%4+1024];\n\t"
        "ld.shared.b32 v0, [%5];\n\t"
        "ld.shared.b32 v8, [%5+1024];\n\t"
        "xor.b32 w0, w0, 0x80808080;\n\t"
        "xor.b32 w8, w8, 0x80808080;\n\t"
        "prmt.b32 a0, w0, 0, 0x4140;\n\t"
        "prmt.b32 a1, w8, 0, 0x4140;\n\t"
        "prmt.b32 a2, w0, 0, 0x4342;\n\t"
        "prmt.b32 a3, w8, 0, 0x4342;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%6,%7}, "
        "{%10,%11,%12,%13};\n\t"
        "xor.b32 v0, v0, 0x80808080;\n\t"
        "xor.b32 v8, v8, 0x80808080;\n\t"
        "prmt.b32 a0, v0, 0, 0x4140;\n\t"
        "prmt.b32 a1, v8, 0, 0x4140;\n\t"
        "prmt.b32 a2, v0, 0, 0x4342;\n\t"
        "prmt.b32 a3, v8, 0, 0x4342;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {c0,c1,c2,c3}, {a0,a1,a2,a3}, {%8,%9}, "
        "{c0,c1,c2,c3};\n\t"
        "fma.rn.f32 %0, %14, c0, %0;\n\t"
        "fma.rn.f32 %1, %14, c1, %1;\n\t"
        "fma.rn.f32 %2, %15, c2, %2;\n\t"
        "fma.rn.f32 %3, %15, c3, %3;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
        : "r"(addr_a), "r"(addr_b), "r"(xa.x), "r"(xa.y), "r"(xb.x), "r"(xb.y), "f"(off[0]),
          "f"(off[1]), "f"(off[2]), "f"(off[3]), "f"(dg), "f"(dg8));
}

// One half of an fp16 pair as fp32 (HI: the upper half).  One asm per half,
// so a block converts only the scale it uses.
template <bool HI>
__device__ __forceinline__ float half_of_pair(uint32_t v)
{
    float f;
    if constexpr (HI)
        asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(v));
    else
        asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(f) : "r"(v));
    return f;
}

__device__ __forceinline__ uint4 lds128_u32(uint32_t addr)
{
    uint4 v;
    asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 lds128_f32(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
    return v;
}

// Per-lane swizzled offsets of the 8 blocks of a chunk row (constant for a
// lane): TMA's 128-byte swizzle XORs the 16-byte granule index with the row
// index mod 8, and row mod 8 == g for every row this lane reads.  For Q8 the
// two 16-byte halves of a block are packed as two 16-bit offsets.  Q2 / Q3's
// 2-bit plane has 64-byte rows under the 64-byte swizzle: a block is 8
// bytes, half of a 16-byte granule, and the granule index (0..3) is XORed
// with bits 7-8 of the offset, (row / 2) mod 4 -- the same for rows g and g+8.
template <int FMT>
__device__ __forceinline__ void lane_swizzle(int g, int (&sw)[8])
{
#pragma unroll
    for (int jb = 0; jb < 8; jb++) {
        if constexpr (FMT == 2 || FMT == 3) {
            sw[jb] = ((((jb >> 1) ^ (g >> 1)) & 3) << 4) | ((jb & 1) << 3);
        } else if constexpr (FMT == 4 || FMT == 5 || FMT == 6) {   // (Q5, Q6: the low-nibble plane)
            sw[jb] = ((jb ^ g) & 7) << 4;
        } else {
            const int jj = jb & 3;
            sw[jb] = ((((2 * jj) ^ g) & 7) << 4) | (((((2 * jj + 1) ^ g) & 7) << 4) << 16);
        }
    }
}

// The x fragments of a chunk: for block jb, xa = x[k..k+3] and xb =
// x[k+16..k+19] with k = k0 + 32 jb + 4t, for batch column g.  `xp` points at
// x[column g][k0 + 4t]; a lane whose column is absent (g >= B) reads a valid
// row instead -- its mma column is garbage and is never stored, which keeps
// every load unconditional.  Only the nblk valid blocks are read.
template <bool COHERENT>
__device__ __forceinline__ void chunk_load_x(const __half *xp, int nblk, uint2 (&xa)[8],
                                             uint2 (&xb)[8])
{
    if (nblk == 8) {
#pragma unroll
        for (int jb = 0; jb < 8; jb++) {
            xa[jb] = ldg64<COHERENT>(xp + 32 * jb);
            xb[jb] = ldg64<COHERENT>(xp + 32 * jb + 16);
        }
    } else {
#pragma unroll
        for (int jb = 0; jb < 8; jb++) {
            if (jb < nblk) {
                xa[jb] = ldg64<COHERENT>(xp + 32 * jb);
                xb[jb] = ldg64<COHERENT>(xp + 32 * jb + 16);
            } else {
                xa[jb] = xb[jb] = make_uint2(0u, 0u);
            }
        }
    }
}

// A whole chunk: 8 blocks (nblk of them valid) for the chunk's kMT m-tiles,
// with the x fragments already loaded.  codes_s / scales_s are the slot's
// shared addresses, laundered through the slot's mbarrier wait.
template <int FMT, int MT>
__device__ __forceinline__ void chunk_mma(uint32_t codes_s, uint32_t scales_s, int nblk, int g,
                                          int t, const int (&sw)[8], const uint2 (&xa)[8],
                                          const uint2 (&xb)[8], float (&acc)[MT][4], uint32_t m16)
{
    uint4 sc[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; mt++) {
        sc[mt][0] = lds128_u32(scales_s + (16 * mt + g) * 16);
        sc[mt][1] = lds128_u32(scales_s + (16 * mt + g + 8) * 16);
    }
    constexpr bool kLow2 = FMT == 2 || FMT == 3;     // first plane: 2-bit, 64-byte rows
    const uint32_t lane_codes = kLow2 ? codes_s + g * 64 + 4 * (t & 1) : codes_s + g * 128 + 4 * t;
    // Q6 / Q5 / Q3: this lane's top-bit group (after the 16 rows of the first
    // plane; rows 64 / 32 / 32 bytes apart) and the multipliers that move its
    // bits into place.
    const uint32_t lane_hi = FMT == 6   ? codes_s + 16 * 128 + g * 64 + 4 * (t & 1)
                             : FMT == 3 ? codes_s + 16 * 64 + g * 32
                                        : codes_s + 16 * 128 + g * 32;
    const uint32_t mh1 = FMT == 6 || kLow2 ? 1u << (8 - 2 * (t >> 1)) : 1u << (8 - t);
    const uint32_t mh2 = FMT == 6 || kLow2 ? 1u << (4 - 2 * (t >> 1)) : 1u << (4 - t);
    const uint32_t mh3 = 1u << (10 - t), mh4 = 1u << (6 - t);    // Q3: bit 2 of a code -> bit 10
    auto one_block = [&](int jb) {
        float off[4];
        block_offset<FMT>(xa[jb], xb[jb], off);
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
            const uint32_t s0 = pick_u32(sc[mt][0], jb >> 1), s8 = pick_u32(sc[mt][1], jb >> 1);
            const float dg = (jb & 1) ? half_of_pair<true>(s0) : half_of_pair<false>(s0);
            const float dg8 = (jb & 1) ? half_of_pair<true>(s8) : half_of_pair<false>(s8);
            if constexpr (FMT == 4) {
                block_q4(lane_codes + mt * 2048 + sw[jb], xa[jb], xb[jb], off, dg, dg8, acc[mt], m16);
            } else if constexpr (kLow2) {
                block_q23<FMT>(lane_codes + sw[jb], lane_hi + 4 * jb, xa[jb], xb[jb], off, dg, dg8,
                               acc[mt], mh1, mh2, mh3, mh4);
            } else if constexpr (FMT == 6 || FMT == 5) {
                block_qtop<FMT>(lane_codes + sw[jb], lane_hi + (FMT == 6 ? 8 : 4) * jb, xa[jb],
                                xb[jb], off, dg, dg8, acc[mt], m16, mh1, mh2);
            } else {
                const uint32_t base = lane_codes + (jb >> 2) * 2048;
                block_q8(base + (sw[jb] & 0xffff), base + (sw[jb] >> 16), xa[jb], xb[jb], off, dg,
                         dg8, acc[mt]);
            }
        }
    };
    if (nblk == 8) {
#pragma unroll
        for (int jb = 0; jb < 8; jb++)
            one_block(jb);
    } else {
#pragma unroll
        for (int jb = 0; jb < 8; jb++)
            if (jb < nblk)
                one_block(jb);
    }
}

}  // namespace bq
