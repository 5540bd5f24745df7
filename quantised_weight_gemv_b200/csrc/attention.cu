// attention.cu -- decode attention over a block-quantised (Q8) KV cache, sm_100a.
//
// Beside the weight GEMV, a decode step runs attention for the one new token
// of each sequence against its preallocated KV cache (gist.science technical
// summary, "Methodologie" -> "Zero-Allocation Decode Loop"; in the follow-up
// paper memory-bound decode still runs on dedicated GEMV and decode-attention
// kernels, romaanj.github.io review, "Method").  Like the GEMV it
// is bound by memory bandwidth: every cached key and value byte of a sequence
// is read once per token.  The cache is block-quantised in the weights' Q8
// format (32-element blocks along the head dimension, fp16 scale, int8
// codes), which halves the bytes of an fp16 cache.
//
//   s_t  = scale * q . K[t]      p = softmax(s over t < len)      o = sum_t p_t V[t]
//
// Layouts (row-major; D = 128):
//   K codes  int8 [B][Hkv][Tmax][D]   position-major rows
//   K scales fp16 [B][Hkv][Tmax][4]
//   V codes  int8 [B][Hkv][D][Tmax]   transposed: row d holds component d of
//                                     every position, so the P.V product reads
//                                     consecutive positions
//   V scales fp16 [B][Hkv][Tmax][4]   scale of position t's 32-block j
//   q        fp16 [B][Hkv*G][D], query head i uses KV head i / G (G <= 8)
//   o        fp32 [B][Hkv*G][D]
//
// Work: a unit is 128 positions of one (sequence, KV head); units are split
// into contiguous ranges, one per CTA (flash-decoding).  In a CTA, warp w
// takes positions 16w .. 16w+15 of every unit, each warp keeping its own
// online-softmax state for the G query heads; the warps' states are merged in
// shared memory, and the CTAs of one (sequence, head) through the workspace
// (the last to arrive merges in CTA order: deterministic).
//
// Both products run on mma.sync m16n8k16 with the cache codes as exact fp16
// operands (code + 128 in the low bits of a 16-bit lane is the subnormal
// (code + 128) 2^-24), so only fp32 accumulation rounds:
//   scores  S[j][t] (M = query heads, N = positions, K = d): A = q, B = key
//           codes; each 32-block's partial product is scaled by the key's
//           block scale in fp32;
//   values  O^T[d][j] (M = d, N = query heads, K = positions): A = value
//           codes (transposed cache rows), B = p * dV * 2^sigma rounded once to
//           fp16.  The accumulator layout of the score product puts each
//           lane's own p values exactly where the value product's B operand
//           wants them (the score columns are assigned to positions so that a
//           lane's four positions are consecutive), so no shuffles.
// sigma (per 32-block of d) is a running power of two that keeps the largest
// p dV 2^sigma in [2^14, 2^15): p <= 1, so no fp16 overflow, and only terms
// 2^28 times smaller than the largest go subnormal.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {
namespace at {

constexpr int D = 128;
constexpr int TP = 128;                   // positions per unit
constexpr int kCW = 8;                    // warps (16 positions each); warp 0 also issues the TMA
constexpr int kThreads = kCW * 32;
constexpr int S = 2;                      // ring slots
constexpr int kMaxG = 8;
constexpr int kKBytes = TP * D;           // 16 KB of key codes
constexpr int kVBytes = D * TP;           // 16 KB of value codes
constexpr int kScBytes = TP * 4 * 2;      // 1 KB of scales
constexpr int kSlot = kKBytes + kVBytes + 2 * kScBytes;
constexpr int kMergeFloats = kCW * kMaxG * D + 2 * kCW * kMaxG;
constexpr int kPartFloats = 2 * kMaxG + kMaxG * D;   // m, l, O of one CTA partial
constexpr int kMaxCtas = 1024;

constexpr size_t smem_bytes()
{
    return 1024 + (size_t)S * kSlot + (size_t)kMergeFloats * 4 + 256;
}

struct Args {
    CUtensorMap tm_k;    // (D bytes, B*Hkv*Tmax rows), box 128 x 128, SW128
    CUtensorMap tm_vt;   // (Tmax bytes, B*Hkv*D rows), box 128 x 128, SW128
    CUtensorMap tm_ks;   // (8 u16, B*Hkv*Tmax/2 rows), box 8 x 64
    CUtensorMap tm_vs;
    const uint16_t *q;
    const int32_t *lens;
    float *o;
    int B, Hkv, G, Tmax, tps;      // tps = Tmax / TP units per sequence
    int U, nctas;
    float s2_scale;                // scale * log2(e) * 2^24
    int *counters;                 // [B * Hkv]
    float *partials;               // [nctas][2][kPartFloats]
    int *status;
};

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void mbar_arrive1(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// 2^e as fp32 for integer e in [-126, 127]
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// The CTA owning unit x (CTA c owns [floor(c U / n), floor((c + 1) U / n))).
__device__ __forceinline__ int owner_of(long long x, int U, int n) { return (int)(((x + 1) * n - 1) / U); }

__global__ void __launch_bounds__(kThreads, 2) attn_decode_kernel(const __grid_constant__ Args a)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ alignas(8) uint64_t bar_full[S], bar_empty[S], bar_merge;
    __shared__ int merge_old;

    uint8_t *sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t ring = smem_u32(sbase);
    float *mrg = reinterpret_cast<float *>(sbase + S * kSlot);     // [kCW][G][D] O, then m, l
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int cta = blockIdx.x;
    const int u0 = (int)((long long)cta * a.U / a.nctas), u1 = (int)((long long)(cta + 1) * a.U / a.nctas);

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; i++) {
            mbar_init(smem_u32(&bar_full[i]), 1);
            mbar_init(smem_u32(&bar_empty[i]), kCW);
        }
        mbar_init(smem_u32(&bar_merge), kCW * 32);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();

    auto fail = [&]() {
        if (a.status)
            atomicOr(a.status, kStatusTimeout);
    };
    // valid positions of sequence `sq` (b * Hkv + h)
    auto seq_len = [&](int sq) { return min(max(a.lens[sq / a.Hkv], 0), a.Tmax); };

    // TMA issue (warp 0, lane 0): the CTA's units that hold a valid position,
    // S ahead of the consumers; a slot is refilled once every warp has
    // released it.
    const uint64_t pol = policy_evict_first();
    int iss_u = u0, issued = 0;
    auto issue_next = [&]() -> bool {      // lane 0 of warp 0 only
        for (; iss_u < u1; iss_u++) {
            const int sq = iss_u / a.tps, tile = iss_u % a.tps;
            if (tile * TP >= seq_len(sq))
                continue;
            const int slot = issued % S;
            if (!mbar_wait_bounded(smem_u32(&bar_empty[slot]), ((issued / S) & 1) ^ 1)) {
                fail();
                return false;
            }
            const uint32_t base = ring + slot * kSlot;
            const uint32_t bar = smem_u32(&bar_full[slot]);
            const int row = sq * a.Tmax + tile * TP;
            mbar_arrive_expect_tx(bar, kSlot);
            tma_load_2d(base, &a.tm_k, bar, 0, row, pol);
            tma_load_2d(base + kKBytes, &a.tm_vt, bar, tile * TP, sq * D, pol);
            tma_load_2d(base + kKBytes + kVBytes, &a.tm_ks, bar, 0, row / 2, pol);
            tma_load_2d(base + kKBytes + kVBytes + kScBytes, &a.tm_vs, bar, 0, row / 2, pol);
            issued++;
            iss_u++;
            return true;
        }
        return true;
    };
    if (warp == 0 && lane == 0)
        for (int k = 0; k < S; k++)
            if (!issue_next())
                break;

    // ----------------------------------------------------- compute warps ----
    const int w = warp;
    int n = 0;            // units consumed (ring index)
    int nmerge = 0;       // phases of the compute warps' barrier used so far
    bool ok = true;
    // All 256 compute threads: arrive, then wait (bounded) for the phase --
    // an mbarrier rather than bar.sync, so a thread that gave up on a timeout
    // cannot leave the others blocked.
    auto sync_compute = [&]() -> bool {
        mbar_arrive1(smem_u32(&bar_merge));
        const bool r = mbar_wait_bounded(smem_u32(&bar_merge), nmerge & 1);
        nmerge++;
        if (!r)
            fail();
        return r;
    };
    for (int u = u0; u < u1 && ok;) {
        const int sq = u / a.tps;
        const int ue = min(u1, (sq + 1) * a.tps);
        const int L = seq_len(sq);
        const int b = sq / a.Hkv, h = sq % a.Hkv;
        // query fragments of head row j = g (rows >= G and g + 8 are zero):
        // k-step ks covers d 16 ks .. 16 ks + 15 with the lane's elements
        // 16 ks + 4 t4 .. + 3 (the mma k-slot permutation of the decode GEMV)
        uint32_t qa[8], qc[8];
        {
            const bool live = g < a.G;
            const uint16_t *qr = a.q + ((size_t)b * a.Hkv * a.G + (size_t)h * a.G + (live ? g : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                uint2 v = live ? *reinterpret_cast<const uint2 *>(qr + 16 * ks + 4 * t4) : make_uint2(0u, 0u);
                qa[ks] = v.x;
                qc[ks] = v.y;
            }
        }
        // the key zero point: -128 2^-24 sum_{d in block} q[j][d], per block
        float koff[4];
#pragma unroll
        for (int blk = 0; blk < 4; blk++) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16(c, qa[2 * blk], 0u, qc[2 * blk], 0u, 0x80808080u, 0x80808080u);
            mma_f16(c, qa[2 * blk + 1], 0u, qc[2 * blk + 1], 0u, 0x80808080u, 0x80808080u);
            koff[blk] = c[0];
        }
        float m_run = -INFINITY, l_run = 0.f;
        float O[8][4], Co[4][4];
#pragma unroll
        for (int mt = 0; mt < 8; mt++)
            O[mt][0] = O[mt][1] = O[mt][2] = O[mt][3] = 0.f;
#pragma unroll
        for (int blk = 0; blk < 4; blk++)
            Co[blk][0] = Co[blk][1] = Co[blk][2] = Co[blk][3] = 0.f;
        int sig[4] = {126, 126, 126, 126};

        for (; u < ue; u++) {
            const int tile = u % a.tps;
            if (tile * TP >= L)
                continue;
            const int slot = n % S;
            if (!mbar_wait_bounded(smem_u32(&bar_full[slot]), (n / S) & 1)) {
                if (lane == 0)
                    fail();
                ok = false;
                break;
            }
            const uint32_t base = ring + slot * kSlot;
            const int pw = tile * TP + 16 * w;        // this warp's first position
            // the unit's largest value scale per 32-block of d (valid
            // positions only), hence its sigma: dmax 2^sigma in [2^14, 2^15)
            int sig_u[4];
            {
                uint32_t mx0 = 0u, mx1 = 0u;          // fp16 bits of blocks (0, 1) and (2, 3)
                const uint32_t vsb = base + kKBytes + kVBytes + kScBytes;
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int p = lane * 4 + k;
                    if (tile * TP + p < L) {
                        mx0 = __vmaxu2(mx0, lds32(vsb + p * 8) & 0x7FFF7FFFu);
                        mx1 = __vmaxu2(mx1, lds32(vsb + p * 8 + 4) & 0x7FFF7FFFu);
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    mx0 = __vmaxu2(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = __vmaxu2(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
#pragma unroll
                for (int blk = 0; blk < 4; blk++) {
                    const uint32_t mxw = blk < 2 ? mx0 : mx1;
                    const unsigned bits = min((blk & 1) ? (mxw >> 16) : (mxw & 0xFFFFu), 0x7BFFu);
                    const float dmax = __half2float(__ushort_as_half((unsigned short)bits));
                    sig_u[blk] = dmax > 0.f ? 141 - ((__float_as_int(dmax) >> 23) & 0xFF) : 126;
                }
            }
            // running sigma: never increases; rescale what was accumulated
#pragma unroll
            for (int blk = 0; blk < 4; blk++) {
                const int sn = min(sig[blk], sig_u[blk]);
                if (sn != sig[blk]) {
                    const float f = pow2i(sn - sig[blk]);
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4++) {
                        O[2 * blk][q4] *= f;
                        O[2 * blk + 1][q4] *= f;
                        Co[blk][q4] *= f;
                    }
                    sig[blk] = sn;
                }
            }
            if (pw < L) {
                // ------------------------------------------- scores ----
                // score column c of n-tile nt is position 4 (c / 2) + c % 2 + 2 nt
                // of the warp's 16, so the lane's two columns of both n-tiles
                // are its positions 4 t4 .. 4 t4 + 3.
                const uint32_t ks_base = base + kKBytes + kVBytes;         // key scales [pos][4]
                const uint32_t vs_base = ks_base + kScBytes;               // value scales
                float s[4];
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    const int r = 16 * w + 4 * (g >> 1) + (g & 1) + 2 * nt;   // key row (B column g)
                    const uint32_t krow = base + r * 128;
                    const int rsw = r & 7;
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                    for (int blk = 0; blk < 4; blk++) {
                        float c[4] = {koff[blk], koff[blk], 0.f, 0.f};
#pragma unroll
                        for (int kk = 0; kk < 2; kk++) {
                            const int ks = 2 * blk + kk;
                            const uint32_t wv = lds32(krow + ((ks ^ rsw) << 4) + 4 * t4) ^ 0x80808080u;
                            mma_f16(c, qa[ks], 0u, qc[ks], 0u, prmt(wv, 0, 0x4140), prmt(wv, 0, 0x4342));
                        }
                        // the lane's columns 2 t4, 2 t4 + 1 are positions p0, p0 + 1
                        const int p0 = 16 * w + 4 * t4 + 2 * nt;
                        unsigned short k0, k1;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(k0) : "r"(ks_base + p0 * 8 + 2 * blk));
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(k1) : "r"(ks_base + (p0 + 1) * 8 + 2 * blk));
                        acc0 = fmaf(__half2float(__ushort_as_half(k0)), c[0], acc0);
                        acc1 = fmaf(__half2float(__ushort_as_half(k1)), c[1], acc1);
                    }
                    s[2 * nt] = acc0;
                    s[2 * nt + 1] = acc1;
                }
                // ------------------------------------- online softmax ----
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int p = pw + 4 * t4 + i;
                    s[i] = p < L ? s[i] * a.s2_scale : -INFINITY;
                    mx = fmaxf(mx, s[i]);
                }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_run, mx);          // finite: position pw < L exists
                const float alpha = ex2(m_run - m_new);          // 0 when m_run = -inf
                float p[4];
                float ps = 0.f;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    p[i] = ex2(s[i] - m_new);                    // 0 for masked positions
                    ps += p[i];
                }
                l_run = l_run * alpha + ps;
                m_run = m_new;
                // O columns are query heads 2 t4, 2 t4 + 1: their alphas
                const float al0 = __shfl_sync(0xffffffffu, alpha, (2 * t4) * 4);
                const float al1 = __shfl_sync(0xffffffffu, alpha, (2 * t4 + 1) * 4);
#pragma unroll
                for (int mt = 0; mt < 8; mt++) {
                    O[mt][0] *= al0;
                    O[mt][1] *= al1;
                    O[mt][2] *= al0;
                    O[mt][3] *= al1;
                }
#pragma unroll
                for (int blk = 0; blk < 4; blk++) {
                    Co[blk][0] *= al0;
                    Co[blk][1] *= al1;
                    Co[blk][2] *= al0;
                    Co[blk][3] *= al1;
                }
                // --------------------------------------------- values ----
                // value scales of the lane's 4 positions (masked: 0)
                uint4 vsc[2];
                vsc[0] = lds128_u32(vs_base + (16 * w + 4 * t4) * 8);
                vsc[1] = lds128_u32(vs_base + (16 * w + 4 * t4 + 2) * 8);
#pragma unroll
                for (int blk = 0; blk < 4; blk++) {
                    const float f = pow2i(sig[blk]);
                    float pv[4];
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const uint4 &vv = vsc[i >> 1];
                        const uint32_t word = (i & 1) ? (blk < 2 ? vv.z : vv.w) : (blk < 2 ? vv.x : vv.y);
                        const unsigned short hb = (blk & 1) ? (unsigned short)(word >> 16) : (unsigned short)(word & 0xFFFFu);
                        const float dv = __half2float(__ushort_as_half(hb));
                        pv[i] = (pw + 4 * t4 + i < L) ? p[i] * (dv * f) : 0.f;
                    }
                    const uint32_t b0 = pack_f16x2(pv[0], pv[1]), b1 = pack_f16x2(pv[2], pv[3]);
                    // zero point: -128 2^-24 sum_t B'[t][j] (every d row equal)
                    mma_f16(Co[blk], 0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u, b0, b1);
#pragma unroll
                    for (int h2 = 0; h2 < 2; h2++) {
                        const int mt = 2 * blk + h2;
                        const int d0 = 16 * mt + g, d8 = d0 + 8;
                        const uint32_t v0 = lds32(base + kKBytes + d0 * 128 + ((w ^ (d0 & 7)) << 4) + 4 * t4) ^ 0x80808080u;
                        const uint32_t v8 = lds32(base + kKBytes + d8 * 128 + ((w ^ (d8 & 7)) << 4) + 4 * t4) ^ 0x80808080u;
                        mma_f16(O[mt], prmt(v0, 0, 0x4140), prmt(v8, 0, 0x4140), prmt(v0, 0, 0x4342),
                                prmt(v8, 0, 0x4342), b0, b1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive1(smem_u32(&bar_empty[slot]));
            n++;
            // warp 0 refills the ring (waits for every warp to release a slot)
            if (warp == 0) {
                bool iok = true;
                if (lane == 0)
                    iok = issue_next();
                if (!__shfl_sync(0xffffffffu, iok ? 1 : 0, 0)) {
                    ok = false;
                    break;
                }
            }
        }
        if (!ok)
            break;
        // --------------------------------------------- warp -> shared ----
        // lane (g, t4) holds O^T for d = 16 mt + g (+ 8), heads 2 t4 (+ 1)
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
        float *Ow = mrg + (size_t)w * kMaxG * D;
        float *mw = mrg + (size_t)kCW * kMaxG * D;
        float *lw = mw + kCW * kMaxG;
#pragma unroll
        for (int mt = 0; mt < 8; mt++) {
            const int blk = mt >> 1;
            const float f = pow2i(24 - sig[blk]);     // codes entered at 2^-24; B' carried 2^sigma
            const int d0 = 16 * mt + g;
            Ow[(2 * t4) * D + d0] = (O[mt][0] + Co[blk][0]) * f;
            Ow[(2 * t4 + 1) * D + d0] = (O[mt][1] + Co[blk][1]) * f;
            Ow[(2 * t4) * D + d0 + 8] = (O[mt][2] + Co[blk][2]) * f;
            Ow[(2 * t4 + 1) * D + d0 + 8] = (O[mt][3] + Co[blk][3]) * f;
        }
        if (t4 == 0) {
            mw[w * kMaxG + g] = m_run;
            lw[w * kMaxG + g] = l_run;
        }
        if (!sync_compute())      // every warp's partial is in shared memory
            break;
        // ------------------------------------------- merge the warps ----
        // thread i of the 256 compute threads: head j = i / 32, d = 4 (i % 32) .. + 3
        const int i = threadIdx.x;
        const int j = i >> 5, d4 = (i & 31) * 4;
        float mstar = -INFINITY;
        for (int ww = 0; ww < kCW; ww++)
            mstar = fmaxf(mstar, mw[ww * kMaxG + j]);
        float lstar = 0.f, ov[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ww = 0; ww < kCW; ww++) {
            const float mwj = mw[ww * kMaxG + j];
            const float f = mwj == -INFINITY ? 0.f : ex2(mwj - mstar);
            lstar += f * lw[ww * kMaxG + j];
#pragma unroll
            for (int k = 0; k < 4; k++)
                ov[k] += f * mrg[((size_t)ww * kMaxG + j) * D + d4 + k];
        }
        const long long su0 = (long long)sq * a.tps;
        const int cf = owner_of(su0, a.U, a.nctas), cl = owner_of(su0 + a.tps - 1, a.U, a.nctas);
        float *out = a.o + ((size_t)b * a.Hkv * a.G + (size_t)h * a.G + j) * D + d4;
        if (cf == cl) {
            if (j < a.G) {
                const float inv = lstar > 0.f ? 1.f / lstar : 0.f;
                *reinterpret_cast<float4 *>(out) = make_float4(ov[0] * inv, ov[1] * inv, ov[2] * inv, ov[3] * inv);
            }
        } else {
            // this CTA's partial (m, l, O) to its slot (0: the sequence of its
            // first unit, 1: of its last); the last CTA merges them in CTA order
            const int my = (sq == u0 / a.tps) ? 0 : 1;
            float *pp = a.partials + ((size_t)cta * 2 + my) * kPartFloats;
            __stcg(reinterpret_cast<float4 *>(pp + 2 * kMaxG + j * D + d4), make_float4(ov[0], ov[1], ov[2], ov[3]));
            if ((i & 31) == 0) {
                __stcg(pp + j, mstar);
                __stcg(pp + kMaxG + j, lstar);
            }
            __threadfence();
            if (!sync_compute())      // the whole partial is stored
                break;
            if (i == 0)
                merge_old = atom_add_acq_rel_gpu(a.counters + sq, 1);
            if (!sync_compute())      // merge_old is published
                break;
            if (merge_old == cl - cf) {
                __threadfence();
                // The partial of CTA c of this sequence: slot 0 if the sequence
                // holds c's first unit, else slot 1.  Every CTA after cf starts
                // inside the sequence, so only cf can hold it in slot 1 (when
                // cf's range starts in an earlier sequence): one division here,
                // none per partial.
                const int cf_slot = (int)((long long)cf * a.U / a.nctas) < sq * a.tps ? 1 : 0;
                auto part = [&](int c) {
                    return a.partials + ((size_t)c * 2 + (c == cf ? cf_slot : 0)) * kPartFloats;
                };
                // One pass over the partials in CTA order, 8 at a time (their loads
                // in flight together), keeping a running maximum: a merge of
                // many partials costs a few L2 round trips, not one per partial.
                float M = -INFINITY, Ls = 0.f, os[4] = {0.f, 0.f, 0.f, 0.f};
                for (int c0 = cf; c0 <= cl; c0 += 8) {
                    float mc[8], lc[8];
                    float4 oc[8];
#pragma unroll
                    for (int k = 0; k < 8; k++) {
                        if (c0 + k <= cl) {
                            const float *pc = part(c0 + k);
                            mc[k] = __ldcg(pc + j);
                            lc[k] = __ldcg(pc + kMaxG + j);
                            oc[k] = __ldcg(reinterpret_cast<const float4 *>(pc + 2 * kMaxG + j * D + d4));
                        } else {
                            mc[k] = -INFINITY;
                            lc[k] = 0.f;
                            oc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
                    float Mb = M;
#pragma unroll
                    for (int k = 0; k < 8; k++)
                        Mb = fmaxf(Mb, mc[k]);
                    if (Mb == -INFINITY)
                        continue;                        // nothing valid so far
                    const float fr = M == -INFINITY ? 0.f : ex2(M - Mb);   // rescale what was summed
                    Ls *= fr;
                    os[0] *= fr;
                    os[1] *= fr;
                    os[2] *= fr;
                    os[3] *= fr;
#pragma unroll
                    for (int k = 0; k < 8; k++) {
                        const float f = mc[k] == -INFINITY ? 0.f : ex2(mc[k] - Mb);
                        Ls += f * lc[k];
                        os[0] += f * oc[k].x;
                        os[1] += f * oc[k].y;
                        os[2] += f * oc[k].z;
                        os[3] += f * oc[k].w;
                    }
                    M = Mb;
                }
                if (j < a.G) {
                    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
                    *reinterpret_cast<float4 *>(out) = make_float4(os[0] * inv, os[1] * inv, os[2] * inv, os[3] * inv);
                }
                // every partial read: clear them, so the workspace is all-zero
                // again when the call ends (calls of any shape may share it)
                if (!sync_compute())
                    break;
                for (int c = cf; c <= cl; c++) {
                    float *pc = part(c);
                    __stcg(reinterpret_cast<float4 *>(pc + 2 * kMaxG + j * D + d4), make_float4(0.f, 0.f, 0.f, 0.f));
                    if ((i & 31) == 0) {
                        __stcg(pc + j, 0.f);
                        __stcg(pc + kMaxG + j, 0.f);
                    }
                }
                if (i == 0)
                    a.counters[sq] = 0;
            }
        }
        if (!sync_compute())          // the merge buffer is free for the next sequence
            break;
        u = ue;
    }
    // drain: every load issued has landed before the CTA may exit
    if (warp == 0 && lane == 0)
        for (int j = max(0, issued - S); j < issued; j++)
            (void)mbar_wait_bounded(smem_u32(&bar_full[j % S]), (j / S) & 1);
}

}  // namespace at

namespace {

int32_t attn_prepare()
{
    static std::atomic<bool> done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire))
        return BQ_OK;
    if (cudaFuncSetAttribute((const void *)at::attn_decode_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)at::smem_bytes()) !=
        cudaSuccess)
        return BQ_ERR_CUDA;
    if (dev >= 0 && dev < 64)
        done[dev].store(true, std::memory_order_release);
    return BQ_OK;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_attn_workspace_bytes(int32_t B, int32_t Hkv)
{
    if (B < 1 || Hkv < 1)
        return 0;
    return align_up((size_t)B * Hkv * sizeof(int), 256) +
           (size_t)at::kMaxCtas * 2 * at::kPartFloats * sizeof(float);
}

extern "C" int32_t bq_attn_decode_q8(const bq_kv_cache *kv, const uint16_t *q, const int32_t *lens,
                                     int32_t B, int32_t Hkv, int32_t G, float scale, float *o,
                                     void *ws, size_t ws_bytes, int32_t *dev_status, void *stream)
{
    if (!kv || !kv->k_codes || !kv->k_scales || !kv->vt_codes || !kv->v_scales || !q || !lens ||
        !o || !ws)
        return BQ_ERR_NULL;
    if (kv->D != at::D || kv->Tmax < at::TP || kv->Tmax % at::TP != 0 || Hkv < 1 || G < 1 ||
        G > at::kMaxG || !(scale == scale))
        return BQ_ERR_SHAPE;
    if (B < 1)
        return BQ_ERR_BATCH;
    if (!aligned16(kv->k_codes) || !aligned16(kv->k_scales) || !aligned16(kv->vt_codes) ||
        !aligned16(kv->v_scales) || !aligned16(q) || !aligned16(o) || !aligned16(ws))
        return BQ_ERR_ALIGN;
    if (ws_bytes < bq_attn_workspace_bytes(B, Hkv))
        return BQ_ERR_WORKSPACE;
    const long long rows = (long long)B * Hkv * kv->Tmax;
    if (rows >= (1LL << 31) || (long long)B * Hkv * at::D >= (1LL << 31))
        return BQ_ERR_SHAPE;
    int32_t st = attn_prepare();
    if (st != BQ_OK)
        return st;
    const int sms = device_sm_count();
    if (sms <= 0)
        return BQ_ERR_CUDA;
    at::Args a;
    memset(&a, 0, sizeof(a));
    const uint64_t kdims[2] = {(uint64_t)at::D, (uint64_t)rows};
    const uint64_t kstr[1] = {(uint64_t)at::D};
    const uint32_t kbox[2] = {128u, (uint32_t)at::TP};
    const uint64_t vdims[2] = {(uint64_t)kv->Tmax, (uint64_t)B * Hkv * at::D};
    const uint64_t vstr[1] = {(uint64_t)kv->Tmax};
    const uint32_t vbox[2] = {128u, (uint32_t)at::D};
    const uint64_t sdims[2] = {8u, (uint64_t)(rows / 2)};
    const uint64_t sstr[1] = {16u};
    const uint32_t sbox[2] = {8u, (uint32_t)(at::TP / 2)};
    if (!encode_tensor_map(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, kv->k_codes, kdims, kstr, kbox,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !encode_tensor_map(&a.tm_vt, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, kv->vt_codes, vdims, vstr,
                           vbox, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !encode_tensor_map(&a.tm_ks, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, kv->k_scales, sdims, sstr,
                           sbox, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE) ||
        !encode_tensor_map(&a.tm_vs, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, kv->v_scales, sdims, sstr,
                           sbox, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE))
        return BQ_ERR_CUDA;
    a.q = q;
    a.lens = lens;
    a.o = o;
    a.B = B;
    a.Hkv = Hkv;
    a.G = G;
    a.Tmax = kv->Tmax;
    a.tps = kv->Tmax / at::TP;
    a.U = B * Hkv * a.tps;
    // CTAs: two per SM when there are units enough.  Below that, one unit
    // a CTA is not the fastest: a sequence's many CTA partials then cost
    // more to merge than a second unit costs to compute, so such launches
    // give every CTA two units (a sequence of one or two units is then one
    // CTA's, with nothing to merge).
    const int full = std::min(2 * sms, at::kMaxCtas);
    a.nctas = a.U > full ? full : std::max(B * Hkv, (a.U + 1) / 2);
    a.s2_scale = scale * 1.4426950408889634f * 16777216.0f;
    a.counters = static_cast<int *>(ws);
    a.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                           align_up((size_t)B * Hkv * sizeof(int), 256));
    a.status = dev_status;
    void *args[] = {&a};
    cudaError_t e = launch_pdl((const void *)at::attn_decode_kernel, dim3(a.nctas), dim3(at::kThreads),
                               at::smem_bytes(), static_cast<cudaStream_t>(stream), args);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
