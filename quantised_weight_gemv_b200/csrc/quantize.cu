// quantize.cu -- block quantisers (host and device) and plane <-> block
// conversions for the Q2-Q6 and Q8 formats (plane <-> block for Q4 / Q8).
//
// Per 32-weight block along K: a = max|w| (fp32); d = fp16 round-to-nearest-
// even of a/127 (Q8) or a/7 (Q4), computed as an IEEE fp32 division; codes
// q = round-half-away-from-zero(w / d) with w / d an IEEE fp32 division by the
// *stored* scale, clamped to [-127, 127] (Q8), or that +8 clamped to [0, 15]
// (Q4); a block whose fp16 scale is zero gets the zero-point code (0 / 8).
// Q4 byte i of a block packs element i (low nibble) and element i+16 (high).
// Q6 (d = a/31, q = round(w/d)+32 clamped to [0, 63], zero-point code 32):
// a row of codes is 3K/4 bytes -- the low nibbles in Q4's layout (block j at
// byte 16j), then the top 2 bits (block j at byte K/2 + 8j; byte i holds
// those of elements i, i+8, i+16, i+24 in bits 0-1, 2-3, 4-5, 6-7).
// Q5 (d = a/15, q = round(w/d)+16 clamped to [0, 31], zero-point code 16):
// rows of 5K/8 bytes -- the low nibbles as Q4, then one top bit per element
// (block j at byte K/2 + 4j; byte i = 0..3 holds that of element i + 4p in
// bit p).
// Q3 (d = a/3, q = round(w/d)+4 clamped to [0, 7], zero-point code 4): rows
// of 3K/8 bytes -- the low 2 bits of each code (block j at byte 8j; byte i
// holds those of elements i, i+8, i+16, i+24 in bits 0-1, 2-3, 4-5, 6-7),
// then bit 2 (block j at byte K/4 + 4j; byte i = 0..3 holds that of element
// i + 4p in bit p).  Q2 (d = a/1, q = round(w/d)+2 clamped to [0, 3], zero-
// point code 2): rows of K/4 bytes, the 2-bit plane alone.
// The pages name the Q4 and Q8 formats (BaseRT abstract: eight formats from
// Q2 to FP16; technical summary "Belangrijkste Bijdragen": evaluation at Q4
// and Q8) without spelling out their bits; the definition above is the one
// the decode GEMV of this library consumes.
#include <cuda_fp16.h>

#include <cmath>
#include <cstring>

#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {
namespace {

// Bytes of a block in a row's first plane (Q2/Q3: the 2-bit plane; Q4-Q6:
// the low-nibble plane; Q8: the codes) and in its second plane (the top bits
// of Q3, Q5, Q6; none otherwise).
template <int FMT>
__host__ __device__ constexpr int lo_block_bytes()
{
    return FMT == 2 || FMT == 3 ? 8 : (FMT == 8 ? 32 : 16);
}
template <int FMT>
__host__ __device__ constexpr int top_block_bytes()
{
    return FMT == 6 ? 8 : (FMT == 5 || FMT == 3 ? 4 : 0);
}

// codes_out: the block's code bytes (first its first-plane bytes, then its
// top-bit bytes; the caller places them in their planes).
template <int FMT>
__host__ __device__ inline void quantize_block(const float *w, uint8_t *codes_out,
                                               uint16_t *scale_out, bool *ok)
{
    constexpr float kLevels = FMT == 2   ? 1.0f
                              : FMT == 3 ? 3.0f
                              : FMT == 4 ? 7.0f
                              : FMT == 5 ? 15.0f
                              : FMT == 6 ? 31.0f
                                         : 127.0f;
    constexpr int kZero = FMT == 2 ? 2 : FMT == 3 ? 4 : FMT == 4 ? 8 : FMT == 5 ? 16 : FMT == 6 ? 32 : 0;
    float a = 0.0f;
    bool finite = true;
    for (int i = 0; i < 32; i++) {
        const float v = w[i];
        if (!(fabsf(v) <= 3.402823466e38f))
            finite = false;
        a = fmaxf(a, fabsf(v));
    }
    float d = 0.0f;
    uint16_t dbits = 0;
    if (finite) {
#ifdef __CUDA_ARCH__
        const float d32 = __fdiv_rn(a, kLevels);
#else
        const float d32 = a / kLevels;
#endif
        const __half dh = __float2half_rn(d32);
        dbits = __half_as_ushort(dh);
        if ((dbits & 0x7c00u) == 0x7c00u) {
            finite = false;
            dbits = 0;
        } else {
            d = __half2float(dh);
        }
    }
    *ok = finite;
    *scale_out = dbits;
    int q[32];
    for (int i = 0; i < 32; i++) {
        if (!finite || d == 0.0f) {
            q[i] = kZero;
            continue;
        }
#ifdef __CUDA_ARCH__
        const float r = roundf(__fdiv_rn(w[i], d));
#else
        const float r = roundf(w[i] / d);
#endif
        if (FMT != 8) {
            const float s = r + (float)kZero;
            const float top = (float)(2 * kZero - 1);
            q[i] = s < 0.0f ? 0 : (s > top ? (int)top : (int)s);
        } else {
            q[i] = r < -127.0f ? -127 : (r > 127.0f ? 127 : (int)r);
        }
    }
    if (FMT == 2 || FMT == 3) {
        for (int i = 0; i < 8; i++)
            codes_out[i] = (uint8_t)((q[i] & 3) | ((q[i + 8] & 3) << 2) | ((q[i + 16] & 3) << 4) |
                                     ((q[i + 24] & 3) << 6));
        if (FMT == 3)
            for (int i = 0; i < 4; i++) {
                int b = 0;
                for (int p = 0; p < 8; p++)
                    b |= (q[i + 4 * p] >> 2) << p;
                codes_out[8 + i] = (uint8_t)b;
            }
    } else if (FMT == 4) {
        for (int i = 0; i < 16; i++)
            codes_out[i] = (uint8_t)(q[i] | (q[i + 16] << 4));
    } else if (FMT == 5) {
        for (int i = 0; i < 16; i++)
            codes_out[i] = (uint8_t)((q[i] & 15) | ((q[i + 16] & 15) << 4));
        for (int i = 0; i < 4; i++) {
            int b = 0;
            for (int p = 0; p < 8; p++)
                b |= (q[i + 4 * p] >> 4) << p;
            codes_out[16 + i] = (uint8_t)b;
        }
    } else if (FMT == 6) {
        for (int i = 0; i < 16; i++)
            codes_out[i] = (uint8_t)((q[i] & 15) | ((q[i + 16] & 15) << 4));
        for (int i = 0; i < 8; i++)
            codes_out[16 + i] = (uint8_t)((q[i] >> 4) | ((q[i + 8] >> 4) << 2) |
                                          ((q[i + 16] >> 4) << 4) | ((q[i + 24] >> 4) << 6));
    } else {
        for (int i = 0; i < 32; i++)
            codes_out[i] = (uint8_t)(int8_t)q[i];
    }
}

// Code bytes of a row: both planes.
template <int FMT>
__host__ __device__ inline size_t row_code_bytes(int K)
{
    return (size_t)(K / 32) * (lo_block_bytes<FMT>() + top_block_bytes<FMT>());
}

template <int FMT>
int32_t quantize_host(const float *w, int32_t N, int32_t K, uint8_t *codes, uint16_t *scales)
{
    if (!w || !codes || !scales)
        return BQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0)
        return BQ_ERR_SHAPE;
    const int nb = K / 32, ldS = bq_scales_ld(K);
    const size_t row_bytes = row_code_bytes<FMT>(K);
    constexpr int kLo = lo_block_bytes<FMT>(), kTop = top_block_bytes<FMT>();
    const size_t lo_row = (size_t)nb * kLo;            // the top plane starts here
    for (int n = 0; n < N; n++) {
        for (int j = nb; j < ldS; j++)
            scales[(size_t)n * ldS + j] = 0;
        for (int j = 0; j < nb; j++) {
            bool ok = true;
            uint8_t *row = codes + (size_t)n * row_bytes;
            uint8_t buf[32];
            quantize_block<FMT>(w + (size_t)n * K + (size_t)j * 32, buf,
                                scales + (size_t)n * ldS + j, &ok);
            memcpy(row + (size_t)j * kLo, buf, kLo);
            if (kTop > 0)
                memcpy(row + lo_row + (size_t)j * kTop, buf + kLo, kTop);
            if (!ok)
                return BQ_ERR_RANGE;
        }
    }
    return BQ_OK;
}

// One thread per block; each thread reads its 128 contiguous input bytes.
template <int FMT>
__global__ void quantize_kernel(const float *__restrict__ w, int N, int K, uint8_t *codes,
                                uint16_t *scales, int *status)
{
    const int nb = K / 32, ldS = (nb + 7) / 8 * 8;
    const long long total = (long long)N * nb;
    const size_t row_bytes = row_code_bytes<FMT>(K);
    const size_t blk_bytes = lo_block_bytes<FMT>();
    for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < total;
         b += (long long)gridDim.x * blockDim.x) {
        const int n = (int)(b / nb), j = (int)(b - (long long)n * nb);
        float v[32];
        const float4 *src = reinterpret_cast<const float4 *>(w + (size_t)n * K + (size_t)j * 32);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float4 f = src[i];
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
        uint8_t out[32];
        uint16_t sc;
        bool ok;
        quantize_block<FMT>(v, out, &sc, &ok);
        if (!ok && status)
            atomicOr(status, kStatusRange);
        uint32_t wv[8];
        memcpy(wv, out, sizeof(wv));
        if (FMT == 2 || FMT == 3) {
            // (Q3: K % 128 == 0: rows keep both planes aligned)
            uint8_t *row = codes + (size_t)n * row_bytes;
            *reinterpret_cast<uint2 *>(row + (size_t)j * 8) = make_uint2(wv[0], wv[1]);
            if (FMT == 3)
                *reinterpret_cast<uint32_t *>(row + (size_t)K / 4 + (size_t)j * 4) = wv[2];
        } else if (FMT == 5 || FMT == 6) {
            // (Q6: K % 64 == 0, Q5: K % 128 == 0: rows keep both planes aligned)
            uint8_t *row = codes + (size_t)n * row_bytes;
            *reinterpret_cast<uint4 *>(row + (size_t)j * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            if (FMT == 6)
                *reinterpret_cast<uint2 *>(row + (size_t)K / 2 + (size_t)j * 8) = make_uint2(wv[4], wv[5]);
            else
                *reinterpret_cast<uint32_t *>(row + (size_t)K / 2 + (size_t)j * 4) = wv[4];
        } else {
            uint4 *dst = reinterpret_cast<uint4 *>(codes + (size_t)n * row_bytes + (size_t)j * blk_bytes);
            dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            if (FMT == 8)
                dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        }
        scales[(size_t)n * ldS + j] = sc;
        if (j == nb - 1)
            for (int p = nb; p < ldS; p++)
                scales[(size_t)n * ldS + p] = 0;
    }
}

template <int FMT>
int32_t quantize_dev(const float *w, int32_t N, int32_t K, void *codes, uint16_t *scales,
                     int32_t *dev_status, void *stream)
{
    if (!w || !codes || !scales)
        return BQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0 || (FMT == 6 && K % 64 != 0) ||
        ((FMT == 5 || FMT == 3) && K % 128 != 0))
        return BQ_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales))
        return BQ_ERR_ALIGN;
    const long long total = (long long)N * (K / 32);
    const int sms = device_sm_count();
    if (sms <= 0)
        return BQ_ERR_CUDA;
    long long grid = (total + 255) / 256;
    if (grid > 32LL * sms)
        grid = 32LL * sms;
    quantize_kernel<FMT><<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        w, N, K, static_cast<uint8_t *>(codes), scales, dev_status);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <int FMT>
int32_t dequantize_host(const void *codes, const uint16_t *scales, int32_t N, int32_t K, float *w)
{
    if (!codes || !scales || !w)
        return BQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0)
        return BQ_ERR_SHAPE;
    const int ldS = bq_scales_ld(K);
    const uint8_t *c = static_cast<const uint8_t *>(codes);
    for (int n = 0; n < N; n++) {
        for (int k = 0; k < K; k++) {
            const float d = __half2float(__ushort_as_half(scales[(size_t)n * ldS + k / 32]));
            int q;
            if (FMT == 2 || FMT == 3) {
                const uint8_t *row = c + (size_t)n * row_code_bytes<FMT>(K);
                const uint8_t lo = row[(k / 32) * 8 + (k % 8)];
                q = (lo >> (2 * ((k % 32) / 8))) & 3;
                if (FMT == 3) {
                    const uint8_t hi = row[(size_t)K / 4 + (k / 32) * 4 + (k % 4)];
                    q |= ((hi >> ((k % 32) / 4)) & 1) << 2;
                }
                q -= FMT == 3 ? 4 : 2;
            } else if (FMT == 4) {
                const uint8_t byte = c[(size_t)n * (K / 2) + (k / 32) * 16 + (k % 16)];
                q = ((k % 32) < 16 ? (byte & 15) : (byte >> 4)) - 8;
            } else if (FMT == 5) {
                const uint8_t *row = c + (size_t)n * (5 * (size_t)K / 8);
                const uint8_t lo = row[(k / 32) * 16 + (k % 16)];
                const uint8_t hi = row[(size_t)K / 2 + (k / 32) * 4 + (k % 4)];
                q = (((k % 32) < 16 ? (lo & 15) : (lo >> 4)) | (((hi >> ((k % 32) / 4)) & 1) << 4)) - 16;
            } else if (FMT == 6) {
                const uint8_t *row = c + (size_t)n * (3 * (size_t)K / 4);
                const uint8_t lo = row[(k / 32) * 16 + (k % 16)];
                const uint8_t hi = row[(size_t)K / 2 + (k / 32) * 8 + (k % 8)];
                q = (((k % 32) < 16 ? (lo & 15) : (lo >> 4)) | (((hi >> (2 * ((k % 32) / 8))) & 3) << 4)) -
                    32;
            } else {
                q = (int8_t)c[(size_t)n * K + k];
            }
            w[(size_t)n * K + k] = d * (float)q;
        }
    }
    return BQ_OK;
}

template <int FMT>
int32_t planes_to_blocks(const void *codes, const uint16_t *scales, int32_t N, int32_t K,
                         uint8_t *blocks)
{
    if (!codes || !scales || !blocks)
        return BQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0)
        return BQ_ERR_SHAPE;
    const int nb = K / 32, ldS = bq_scales_ld(K);
    const size_t cb = FMT == 4 ? 16 : 32, rec = cb + 2;
    const uint8_t *c = static_cast<const uint8_t *>(codes);
    for (int n = 0; n < N; n++)
        for (int j = 0; j < nb; j++) {
            uint8_t *r = blocks + ((size_t)n * nb + j) * rec;
            const uint16_t s = scales[(size_t)n * ldS + j];
            r[0] = (uint8_t)(s & 0xff);
            r[1] = (uint8_t)(s >> 8);
            memcpy(r + 2, c + ((size_t)n * nb + j) * cb, cb);
        }
    return BQ_OK;
}

template <int FMT>
int32_t blocks_to_planes(const uint8_t *blocks, int32_t N, int32_t K, void *codes, uint16_t *scales)
{
    if (!codes || !scales || !blocks)
        return BQ_ERR_NULL;
    if (N < 1 || K < 32 || K % 32 != 0)
        return BQ_ERR_SHAPE;
    const int nb = K / 32, ldS = bq_scales_ld(K);
    const size_t cb = FMT == 4 ? 16 : 32, rec = cb + 2;
    uint8_t *c = static_cast<uint8_t *>(codes);
    for (int n = 0; n < N; n++) {
        for (int j = 0; j < ldS; j++)
            scales[(size_t)n * ldS + j] = 0;
        for (int j = 0; j < nb; j++) {
            const uint8_t *r = blocks + ((size_t)n * nb + j) * rec;
            scales[(size_t)n * ldS + j] = (uint16_t)(r[0] | (r[1] << 8));
            memcpy(c + ((size_t)n * nb + j) * cb, r + 2, cb);
        }
    }
    return BQ_OK;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" int32_t bq_quantize_q8(const float *w, int32_t N, int32_t K, int8_t *codes,
                                  uint16_t *scales)
{
    return quantize_host<8>(w, N, K, reinterpret_cast<uint8_t *>(codes), scales);
}
extern "C" int32_t bq_quantize_q4(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                  uint16_t *scales)
{
    return quantize_host<4>(w, N, K, codes, scales);
}
extern "C" int32_t bq_dequantize_q8(const int8_t *codes, const uint16_t *scales, int32_t N,
                                    int32_t K, float *w)
{
    return dequantize_host<8>(codes, scales, N, K, w);
}
extern "C" int32_t bq_dequantize_q4(const uint8_t *codes, const uint16_t *scales, int32_t N,
                                    int32_t K, float *w)
{
    return dequantize_host<4>(codes, scales, N, K, w);
}
extern "C" int32_t bq_planes_to_blocks_q4(const uint8_t *codes, const uint16_t *scales, int32_t N,
                                          int32_t K, uint8_t *blocks)
{
    return planes_to_blocks<4>(codes, scales, N, K, blocks);
}
extern "C" int32_t bq_planes_to_blocks_q8(const int8_t *codes, const uint16_t *scales, int32_t N,
                                          int32_t K, uint8_t *blocks)
{
    return planes_to_blocks<8>(codes, scales, N, K, blocks);
}
extern "C" int32_t bq_blocks_to_planes_q4(const uint8_t *blocks, int32_t N, int32_t K,
                                          uint8_t *codes, uint16_t *scales)
{
    return blocks_to_planes<4>(blocks, N, K, codes, scales);
}
extern "C" int32_t bq_blocks_to_planes_q8(const uint8_t *blocks, int32_t N, int32_t K,
                                          int8_t *codes, uint16_t *scales)
{
    return blocks_to_planes<8>(blocks, N, K, codes, scales);
}
extern "C" int32_t bq_quantize_q2(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                  uint16_t *scales)
{
    return quantize_host<2>(w, N, K, codes, scales);
}
extern "C" int32_t bq_dequantize_q2(const uint8_t *codes, const uint16_t *scales, int32_t N,
                                    int32_t K, float *w)
{
    return dequantize_host<2>(codes, scales, N, K, w);
}
extern "C" int32_t bq_quantize_q2_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                      uint16_t *scales, int32_t *dev_status, void *stream)
{
    return quantize_dev<2>(w, N, K, codes, scales, dev_status, stream);
}
extern "C" int32_t bq_quantize_q3(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                  uint16_t *scales)
{
    return quantize_host<3>(w, N, K, codes, scales);
}
extern "C" int32_t bq_dequantize_q3(const uint8_t *codes, const uint16_t *scales, int32_t N,
                                    int32_t K, float *w)
{
    return dequantize_host<3>(codes, scales, N, K, w);
}
extern "C" int32_t bq_quantize_q3_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                      uint16_t *scales, int32_t *dev_status, void *stream)
{
    return quantize_dev<3>(w, N, K, codes, scales, dev_status, stream);
}
extern "C" int32_t bq_quantize_q5(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                  uint16_t *scales)
{
    return quantize_host<5>(w, N, K, codes, scales);
}
extern "C" int32_t bq_dequantize_q5(const uint8_t *codes, const uint16_t *scales, int32_t N,
                                    int32_t K, float *w)
{
    return dequantize_host<5>(codes, scales, N, K, w);
}
extern "C" int32_t bq_quantize_q5_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                      uint16_t *scales, int32_t *dev_status, void *stream)
{
    return quantize_dev<5>(w, N, K, codes, scales, dev_status, stream);
}
extern "C" int32_t bq_quantize_q6(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                  uint16_t *scales)
{
    return quantize_host<6>(w, N, K, codes, scales);
}
extern "C" int32_t bq_dequantize_q6(const uint8_t *codes, const uint16_t *scales, int32_t N,
                                    int32_t K, float *w)
{
    return dequantize_host<6>(codes, scales, N, K, w);
}
extern "C" int32_t bq_quantize_q6_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                      uint16_t *scales, int32_t *dev_status, void *stream)
{
    return quantize_dev<6>(w, N, K, codes, scales, dev_status, stream);
}
extern "C" int32_t bq_quantize_q4_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                                      uint16_t *scales, int32_t *dev_status, void *stream)
{
    return quantize_dev<4>(w, N, K, codes, scales, dev_status, stream);
}
extern "C" int32_t bq_quantize_q8_dev(const float *w, int32_t N, int32_t K, int8_t *codes,
                                      uint16_t *scales, int32_t *dev_status, void *stream)
{
    return quantize_dev<8>(w, N, K, codes, scales, dev_status, stream);
}
