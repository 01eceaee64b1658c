// The block-int4 dequantisation of the frozen weights.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "f32x2.cuh"

namespace lmlp {

// x / 7 correctly rounded in fp32 for x = fp32(q) * fp32(scale), q an int4
// code and scale an fp16 (so x has at most 14 significant bits): the product
// y = x * fl(1/7), then one correction by the exact residual e = x - 7y,
// y + e * fl(1/7) rounded once by the FMA.  Checked exhaustively with exact
// rational arithmetic against the correctly rounded quotient for every code
// 1..8 and every positive finite fp16 scale (253,944 cases); negative x
// follow from the sign symmetry of round-to-nearest-even.  It is evaluated
// from -x (y = (-x)(-1/7), e' = 7y + (-x) = -e, result = e'(-1/7) + y): the
// same values, and a zero x keeps its sign (a residual sum of +0 and -0
// would otherwise turn -0 into +0).  Two lanes at a time; neg_x = -x.
__device__ __forceinline__ uint64_t div7_rn_neg2(uint64_t neg_x) {
    const uint64_t nr = f2_packf(-1.0f / 7.0f, -1.0f / 7.0f);  // -fl(1/7)
    const uint64_t seven = f2_packf(7.0f, 7.0f);
    const uint64_t y = f2_mul(neg_x, nr);
    const uint64_t e = f2_fma(y, seven, neg_x);
    return f2_fma(e, nr, y);
}

// prmt: byte k of the result is byte (c >> 4k) & 7 of {b, a} (a's bytes
// 0-3, then b's), or, when bit 3 of that selector nibble is set, that
// byte's sign bit replicated over all eight bits.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// The sixteen bf16 values one block-int4 scale gives, as byte tables for
// prmt lookups.  Code nibble n (two's complement, q = n or n - 16) takes
//   T[n] = bf16_rne(fl(q * scale) / 7),
// which for n >= 8 is -T'[16 - n] with T'[m] = bf16_rne(fl(m * scale) / 7):
// q * scale is exact in fp32 and round-to-nearest-even is symmetric, so the
// nine quotients m = 0..8 give every value.  lo[0], lo[1] hold the low bytes
// of T[0..7], lo[2], lo[3] those of T[8..15]; hi likewise the high bytes.
struct Int4Lut {
    uint32_t lo[4], hi[4];
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ Int4Lut int4_lut(float scale) {
    float y[10];
    if (fabsf(scale) <= 65504.0f) {
        // finite: the exact products m * scale, divided by 7 with the
        // correctly rounded sequence div7_rn_neg2, two quotients per step
        const uint64_t ns2 = f2_packf(-scale, -scale);
#pragma unroll
        for (int m = 0; m < 10; m += 2) {
            const uint64_t q2 = div7_rn_neg2(f2_mul(f2_packf(static_cast<float>(m), static_cast<float>(m + 1)), ns2));
            f2_unpack(q2, y[m], y[m + 1]);
        }
    } else {
        // inf or NaN: IEEE's own multiply and divide (0 * inf is NaN)
#pragma unroll
        for (int m = 0; m < 10; ++m) y[m] = __fdiv_rn(static_cast<float>(m) * scale, 7.0f);
    }
    const uint32_t p01 = bf16x2_bits(y[0], y[1]), p23 = bf16x2_bits(y[2], y[3]);
    const uint32_t p45 = bf16x2_bits(y[4], y[5]), p67 = bf16x2_bits(y[6], y[7]);
    const uint32_t n87 = bf16x2_bits(y[8], y[7]), n65 = bf16x2_bits(y[6], y[5]);
    const uint32_t n43 = bf16x2_bits(y[4], y[3]), n21 = bf16x2_bits(y[2], y[1]);
    Int4Lut t;
    t.lo[0] = prmt(p01, p23, 0x6420u);
    t.hi[0] = prmt(p01, p23, 0x7531u);
    t.lo[1] = prmt(p45, p67, 0x6420u);
    t.hi[1] = prmt(p45, p67, 0x7531u);
    t.lo[2] = prmt(n87, n65, 0x6420u);               // codes 8..11: magnitudes 8, 7, 6, 5
    t.hi[2] = prmt(n87, n65, 0x7531u) ^ 0x80808080u;  // negated: sign bit of the high byte
    t.lo[3] = prmt(n43, n21, 0x6420u);               // codes 12..15: magnitudes 4, 3, 2, 1
    t.hi[3] = prmt(n43, n21, 0x7531u) ^ 0x80808080u;
    return t;
}

// Eight codes (one 4-byte word, element e in nibble e) -> eight bf16 values
// (16 bytes, element e at bytes 2e, 2e + 1), by table lookup: the low three
// bits of each nibble pick a byte of the code-0..7 or the code-8..15 table,
// and the nibble's bit 3 picks the table.
__device__ __forceinline__ uint4 int4_expand8(uint32_t w, const Int4Lut& t) {
    const uint32_t sel = w & 0x77777777u;
    const uint32_t w4 = w << 4;
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sh = h ? sel >> 16 : sel;
        // 0xFF for the elements whose code is negative: the sign bit of
        // nibble e is the top bit of a byte of w << 4 (e even) or of w (e odd)
        const uint32_t neg = prmt(w4, w, h ? 0xFBEAu : 0xD9C8u);
        const uint32_t lo = (prmt(t.lo[0], t.lo[1], sh) & ~neg) | (prmt(t.lo[2], t.lo[3], sh) & neg);
        const uint32_t hi = (prmt(t.hi[0], t.hi[1], sh) & ~neg) | (prmt(t.hi[2], t.hi[3], sh) & neg);
        o[2 * h] = prmt(lo, hi, 0x5140u);      // elements 4h, 4h + 1
        o[2 * h + 1] = prmt(lo, hi, 0x7362u);  // elements 4h + 2, 4h + 3
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// One 64-element block ("line"): 32 bytes of codes -> 128 bytes of bf16.
__device__ __forceinline__ void int4_line(uint4 c0, uint4 c1, float scale, uint4 (&out)[8]) {
    const Int4Lut t = int4_lut(scale);
    out[0] = int4_expand8(c0.x, t);
    out[1] = int4_expand8(c0.y, t);
    out[2] = int4_expand8(c0.z, t);
    out[3] = int4_expand8(c0.w, t);
    out[4] = int4_expand8(c1.x, t);
    out[5] = int4_expand8(c1.y, t);
    out[6] = int4_expand8(c1.z, t);
    out[7] = int4_expand8(c1.w, t);
}

// The standalone dequantisation: one thread per line.  Codes [rows, cols/2]
// and scales [rows, cols/64] are row-major, so line L (elements 64L ..) is
// code bytes 32L .., scale L and output bytes 128L ..; the GEMMs' dequant
// warps run the same int4_line on their stage's lines.
constexpr int kDqThreads = 128;

__global__ void __launch_bounds__(kDqThreads) dequant_int4_kernel(const uint4* __restrict__ packed,
                                                                  const __half* __restrict__ scales,
                                                                  long long nlines, uint4* __restrict__ w) {
    for (long long L = static_cast<long long>(blockIdx.x) * kDqThreads + threadIdx.x; L < nlines;
         L += static_cast<long long>(gridDim.x) * kDqThreads) {
        const uint4 c0 = __ldcs(packed + 2 * L), c1 = __ldcs(packed + 2 * L + 1);
        uint4 o[8];
        int4_line(c0, c1, __half2float(scales[L]), o);
#pragma unroll
        for (int q = 0; q < 8; ++q) __stcs(w + 8 * L + q, o[q]);
    }
}

// ---------------------------------------------------------------- FP8 (E4M3)

// Four codes (one 4-byte word, element e in byte e) -> four bf16 values
// bf16_rne(fp32(e4m3) * scale): the f16 values widen exactly to fp32, one
// fp32 multiply per element (two lanes per instruction), one rounding to
// bf16.  s2 = {scale, scale}.
__device__ __forceinline__ uint2 fp8_expand4(uint32_t w, uint64_t s2) {
    uint32_t h01, h23;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(h01), "=r"(h23)
        : "r"(w));
    float f0, f1, f2, f3;
    asm("{\n\t.reg .b16 a, b, c, d;\n\tmov.b32 {a, b}, %4;\n\tmov.b32 {c, d}, %5;\n\t"
        "cvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\tcvt.f32.f16 %2, c;\n\tcvt.f32.f16 %3, d;\n\t}"
        : "=f"(f0), "=f"(f1), "=f"(f2), "=f"(f3)
        : "r"(h01), "r"(h23));
    float p0, p1, p2, p3;
    f2_unpack(f2_mul(f2_packf(f0, f1), s2), p0, p1);
    f2_unpack(f2_mul(f2_packf(f2, f3), s2), p2, p3);
    return make_uint2(bf16x2_bits(p0, p1), bf16x2_bits(p2, p3));
}

// One 64-element line: 64 code bytes (c[0] holds elements 0..15) -> 128
// bytes of bf16 (out[q] holds elements 8q .. 8q + 7).
__device__ __forceinline__ void fp8_line(const uint4 (&c)[4], float scale, uint4 (&out)[8]) {
    const uint64_t s2 = f2_packf(scale, scale);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint2 a = fp8_expand4(c[i].x, s2), b = fp8_expand4(c[i].y, s2);
        const uint2 e = fp8_expand4(c[i].z, s2), f = fp8_expand4(c[i].w, s2);
        out[2 * i] = make_uint4(a.x, a.y, b.x, b.y);
        out[2 * i + 1] = make_uint4(e.x, e.y, f.x, f.y);
    }
}

// The standalone FP8 dequantisation, one thread per line: codes [rows, cols]
// and scales [rows, cols/64] (fp32) row-major, so line L is code bytes 64L ..,
// scale L and output bytes 128L ..  The GEMMs' dequant warps run the same
// fp8_line on their stage's lines.
__global__ void __launch_bounds__(kDqThreads) dequant_fp8_kernel(const uint4* __restrict__ codes,
                                                                 const float* __restrict__ scales,
                                                                 long long nlines, uint4* __restrict__ w) {
    for (long long L = static_cast<long long>(blockIdx.x) * kDqThreads + threadIdx.x; L < nlines;
         L += static_cast<long long>(gridDim.x) * kDqThreads) {
        uint4 c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) c[i] = __ldcs(codes + 4 * L + i);
        uint4 o[8];
        fp8_line(c, scales[L], o);
#pragma unroll
        for (int q = 0; q < 8; ++q) __stcs(w + 8 * L + q, o[q]);
    }
}

// Block scales [rows, nb] (nb = cols / 64) -> their transpose [nb, rows], so
// that the scales of one 64-column block of consecutive rows are contiguous
// and a GEMM stage can fetch them with one TMA box.  Up to three matrices per
// launch (blockIdx.y); a CTA takes a strip of 32 rows and walks its 32 x 32
// tiles through shared memory (reads along a row, writes along a column of
// the transpose, both coalesced).
template <class T>
struct ScaleT {
    const T* src[3];
    T* dst[3];
    int rows[3], nb[3];
};

template <class T>
__global__ void __launch_bounds__(256) scale_transpose_kernel(const ScaleT<T> a) {
    __shared__ T tile[32][33];
    const int z = blockIdx.y;
    const int rows = a.rows[z], nb = a.nb[z];
    const int r0 = blockIdx.x * 32;
    if (r0 >= rows) return;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
    for (int b0 = 0; b0 < nb; b0 += 32) {
        for (int i = ty; i < 32; i += 8) {
            const int r = r0 + i, b = b0 + tx;
            if (r < rows && b < nb) tile[i][tx] = a.src[z][static_cast<long long>(r) * nb + b];
        }
        __syncthreads();
        for (int i = ty; i < 32; i += 8) {
            const int b = b0 + i, r = r0 + tx;
            if (r < rows && b < nb) a.dst[z][static_cast<long long>(b) * rows + r] = tile[tx][i];
        }
        __syncthreads();
    }
}

}  // namespace lmlp
