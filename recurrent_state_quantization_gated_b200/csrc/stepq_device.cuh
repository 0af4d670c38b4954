// stepq_device.cuh -- device building blocks shared by the libstepq kernels (sm_100a).
//
// Tile mapping (one (sequence, head) state tile of D x D, D = 64 or 128, row = key channel i,
// column = value channel j): a thread owns CPL adjacent columns (lane % LPR) of RPT rows.
// LPR = D/CPL lanes span one row; a warp covers RPW = 32/LPR rows per instruction; warp w owns
// the rows (slots) [w*RPT*RPW, (w+1)*RPT*RPW). The fused decode kernel uses CPL = 8 so that
// the per-row work (metadata, constants, addresses) is shared by eight elements; the state
// conversion and comparison kernels use CPL = 4.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace stepq {

constexpr float kHalfMinNormal = 6.103515625e-05f;   // 2^-14
constexpr float kHalfMax = 65504.0f;
constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23: x + M rounds x to an integer
constexpr uint32_t kRoundMagicBits = 0x4B400000u;
constexpr float kTwo23 = 8388608.0f;                  // 2^23

template <int D, int CPL = 4>
struct Map {
    static constexpr int kCols = CPL;
    static constexpr int kThreads = (D == 128) ? 256 : 128;
    static constexpr int kMinBlocks = (D == 128) ? 2 : 4;          // keeps registers <= 128
    static constexpr int kWarps = kThreads / 32;
    static constexpr int LPR = D / CPL;                // lanes per row
    static constexpr int RPW = 32 / LPR;               // rows per warp instruction
    static constexpr int RPT = D / (kWarps * RPW);     // rows per thread
    static constexpr int kRowsPerWarp = RPT * RPW;
    __device__ static int col_lane(int lane) { return lane % LPR; }
    __device__ static int sub_row(int lane) { return lane / LPR; }
    __device__ static int row(int warp, int lane, int r) {
        return warp * kRowsPerWarp + r * RPW + sub_row(lane);
    }
};

// ------------------------------------------------------------------------------------------
// small numeric helpers
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ int qmax_of(int b) { return (1 << (b - 1)) - 1; }
__device__ __forceinline__ float znorm_of(int b) { return __int_as_float((127 + 8 - b) << 23); }  // 2^(8-b)
// 1/q_b for b in {2, 4, 6, 8}, correctly rounded.
__device__ __forceinline__ float inv_qmax_of(int b) {
    return b == 2 ? 1.0f : b == 4 ? 1.0f / 7.0f : b == 6 ? 1.0f / 31.0f : 1.0f / 127.0f;
}

// A positive scale to binary16: clamp into [2^-14, 65504] (NaN -> floor), round to nearest even.
__device__ __forceinline__ __half scale_to_half(float x) {
    x = fminf(fmaxf(x, kHalfMinNormal), kHalfMax);   // fmaxf(NaN, a) = a
    return __float2half_rn(x);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ------------------------------------------------------------------------------------------
// packed codes: the 4 adjacent columns (4cl .. 4cl+3) of one row at width b.
// Codes are b-bit two's complement. 2- and 8-bit rows keep column j at bit j*b; a 4-bit row
// (and the low plane of a 6-bit row) keeps the four columns of each 16-bit group in nibble
// order 0, 2, 1, 3, i.e. column 4cl+m at bit 4*{0,2,1,3}[m] of halfword cl; a 6-bit row is
// the low-nibble plane (D/2 bytes) followed by the high-crumb plane (D/4 bytes).
//
// Unpacking ORs (sign-flipped) fields into the mantissa of 2^23 so that each field becomes an
// exact float 2^23 + (q + 2^(b-1)) 2^p, p its bit position; one fused multiply-add by 2^-p
// then yields q exactly. Packing reads q from the low bits of the float M + q (M = 1.5 2^23).
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 bits2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }

// Four codes held in registers -> exact floats. lo: the four fields at their canonical bit
// positions (8-bit: bytes 0..3; 4-bit: nibbles at bits 0, 8, 4, 12; 2-bit: crumbs at 0, 2, 4,
// 6; 6-bit: the low nibbles as for 4-bit); hi: the high crumbs of a 6-bit row (bits 0..7).
// Bits outside those positions are ignored.
// (a & M) | c in one logic instruction (the compiler's own lowering of this pattern takes two).
template <uint32_t M>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(M), "r"(c));
    return d;
}

// Sign-bit flips that turn the b-bit two's complement fields of a code word into offset binary
// (field + 2^(b-1)): applied once per word before the per-field float construction below.
template <int BW>
__device__ __forceinline__ uint32_t flip_signs(uint32_t w) {
    if constexpr (BW == 8) return w ^ 0x80808080u;
    else if constexpr (BW == 4) return w ^ 0x88888888u;
    else return w ^ 0xAAAAAAAAu;   // 2-bit fields, and the high-crumb plane of 6-bit rows
}

// Four codes as floats (exact small integers): fields of lo (and for b = 6 the high crumbs in
// hi), both already passed through flip_signs. Each field is masked into the mantissa of 2^23
// (one logic instruction), then one paired FMA removes the offset and the field's place value.
template <int BW>
__device__ __forceinline__ void unpack4f(uint32_t lo, uint32_t hi, float2& z01, float2& z23) {
    constexpr uint32_t F = 0x4B000000u;   // bits of 2^23
    if constexpr (BW == 8) {
        const float2 c = make_float2(-(kTwo23 + 128.0f), -(kTwo23 + 128.0f));
        z01 = add2(bits2(__byte_perm(lo, F, 0x7650), __byte_perm(lo, F, 0x7651)), c);
        z23 = add2(bits2(__byte_perm(lo, F, 0x7652), __byte_perm(lo, F, 0x7653)), c);
    } else if constexpr (BW == 4) {
        z01 = fma2(bits2(and_or<0x000Fu>(lo, F), and_or<0x0F00u>(lo, F)),
                   make_float2(1.0f, 0x1p-8f), make_float2(-(kTwo23 + 8.0f), -(0x1p15f + 8.0f)));
        z23 = fma2(bits2(and_or<0x00F0u>(lo, F), and_or<0xF000u>(lo, F)),
                   make_float2(0x1p-4f, 0x1p-12f), make_float2(-(0x1p19f + 8.0f), -(0x1p11f + 8.0f)));
    } else if constexpr (BW == 2) {
        z01 = fma2(bits2(and_or<0x03u>(lo, F), and_or<0x0Cu>(lo, F)),
                   make_float2(1.0f, 0x1p-2f), make_float2(-(kTwo23 + 2.0f), -(0x1p21f + 2.0f)));
        z23 = fma2(bits2(and_or<0x30u>(lo, F), and_or<0xC0u>(lo, F)),
                   make_float2(0x1p-4f, 0x1p-6f), make_float2(-(0x1p19f + 2.0f), -(0x1p17f + 2.0f)));
    } else {  // 6: z = lo + 16 (hi - 2), hi = sign-flipped high crumb, both taken exactly
        const float2 h01 = fma2(bits2(and_or<0x03u>(hi, F), and_or<0x0Cu>(hi, F)),
                                make_float2(16.0f, 4.0f), make_float2(-142606368.0f, -33587232.0f));
        const float2 h23 = fma2(bits2(and_or<0x30u>(hi, F), and_or<0xC0u>(hi, F)),
                                make_float2(1.0f, 0.25f), make_float2(-8912928.0f, -2099232.0f));
        z01 = fma2(bits2(and_or<0x000Fu>(lo, F), and_or<0x0F00u>(lo, F)), make_float2(1.0f, 0x1p-8f), h01);
        z23 = fma2(bits2(and_or<0x00F0u>(lo, F), and_or<0xF000u>(lo, F)), make_float2(0x1p-4f, 0x1p-12f), h23);
    }
}

// As unpack4f, from the stored (two's complement) code words.
template <int BW>
__device__ __forceinline__ void unpack4r(uint32_t lo, uint32_t hi, float2& z01, float2& z23) {
    if constexpr (BW == 6) unpack4f<6>(lo, flip_signs<2>(hi), z01, z23);
    else unpack4f<BW>(flip_signs<BW>(lo), 0u, z01, z23);
}

// The CPL = 4 chunk of one row (lane cl owns columns 4cl .. 4cl+3).
template <int D, int BW>
__device__ __forceinline__ void unpack4(const uint8_t* row, int cl, float2& z01, float2& z23) {
    if constexpr (BW == 8) unpack4r<8>(*reinterpret_cast<const uint32_t*>(row + 4 * cl), 0u, z01, z23);
    else if constexpr (BW == 4) unpack4r<4>(*reinterpret_cast<const uint16_t*>(row + 2 * cl), 0u, z01, z23);
    else if constexpr (BW == 2) unpack4r<2>(row[cl], 0u, z01, z23);
    else unpack4r<6>(*reinterpret_cast<const uint16_t*>(row + 2 * cl), row[D / 2 + cl], z01, z23);
}

// The code words of one CPL = 8 row chunk, loaded ahead of unpacking: x / y hold the 8-bit
// row's two words, the 6-bit row's low plane word and high plane halfword, or the 4- and 2-bit
// rows' single word (y unused).
template <int D, int BW>
__device__ __forceinline__ uint2 load8(const uint8_t* row, int cl) {
    if constexpr (BW == 8) return *reinterpret_cast<const uint2*>(row + 8 * cl);
    else if constexpr (BW == 4) return make_uint2(*reinterpret_cast<const uint32_t*>(row + 4 * cl), 0u);
    else if constexpr (BW == 2) return make_uint2(*reinterpret_cast<const uint16_t*>(row + 2 * cl), 0u);
    else return make_uint2(*reinterpret_cast<const uint32_t*>(row + 4 * cl),
                           *reinterpret_cast<const uint16_t*>(row + D / 2 + 2 * cl));
}

// The eight codes of a CPL = 8 chunk from its code words (one sign flip per word).
template <int BW>
__device__ __forceinline__ void unpack8r(uint2 w, float2 z[4]) {
    if constexpr (BW == 8) {
        unpack4f<8>(flip_signs<8>(w.x), 0u, z[0], z[1]);
        unpack4f<8>(flip_signs<8>(w.y), 0u, z[2], z[3]);
    } else if constexpr (BW == 4) {
        const uint32_t u = flip_signs<4>(w.x);
        unpack4f<4>(u, 0u, z[0], z[1]);
        unpack4f<4>(u >> 16, 0u, z[2], z[3]);
    } else if constexpr (BW == 2) {
        const uint32_t u = flip_signs<2>(w.x);
        unpack4f<2>(u, 0u, z[0], z[1]);
        unpack4f<2>(u >> 8, 0u, z[2], z[3]);
    } else {
        const uint32_t h = flip_signs<2>(w.y);
        unpack4f<6>(w.x, h, z[0], z[1]);
        unpack4f<6>(w.x >> 16, h >> 8, z[2], z[3]);
    }
}

// The CPL = 8 chunk of one row (lane cl owns columns 8cl .. 8cl+7): one load per plane.
template <int D, int BW>
__device__ __forceinline__ void unpack8(const uint8_t* row, int cl, float2 z[4]) {
    unpack8r<BW>(load8<D, BW>(row, cl), z);
}

// max(|a|, |b|, |c|) in one instruction.
__device__ __forceinline__ float max_abs3(float a, float b, float c) {
    float d;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Reciprocal by the special-function unit (about one ulp; inputs are normal and positive).
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint32_t vmax_s16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t vmin_s16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Bytes q0..q3 from four words holding q in their low 16 bits (e.g. the bits of M + q,
// |q| < 2^15); with CLAMP the codes are first limited to [-q_b, q_b], two at a time.
template <int BW, bool CLAMP>
__device__ __forceinline__ uint32_t gather4(uint32_t zq0, uint32_t zq1, uint32_t zq2, uint32_t zq3) {
    uint32_t p01 = __byte_perm(zq0, zq1, 0x5410);
    uint32_t p23 = __byte_perm(zq2, zq3, 0x5410);
    if constexpr (CLAMP) {
        constexpr uint32_t qb = (1u << (BW - 1)) - 1u;
        constexpr uint32_t hi = qb | (qb << 16);
        constexpr uint32_t lo = ((0x10000u - qb) & 0xFFFFu) | ((0x10000u - qb) << 16);
        p01 = vmin_s16x2(vmax_s16x2(p01, lo), hi);
        p23 = vmin_s16x2(vmax_s16x2(p23, lo), hi);
    }
    return __byte_perm(p01, p23, 0x6420);
}

// Packed fields of four codes given as bytes t = q0 | q1 << 8 | q2 << 16 | q3 << 24.
__device__ __forceinline__ uint32_t nibbles4(uint32_t t) {   // (t & 0x0F0F) | ((t >> 12) & 0xF0F0), 16 bits
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(t), "r"(t >> 12), "n"(0x0F0F0F0Fu));
    return d;
}
__device__ __forceinline__ uint32_t crumbs4(uint32_t t) { return __umulhi((t << 4) & 0x30303030u, 0x10410400u); }  // low byte
__device__ __forceinline__ uint32_t high_crumbs4(uint32_t t) { return __umulhi(t & 0x30303030u, 0x10410400u); }  // low byte

// Store 4 codes (CPL = 4 chunk) at width BW.
template <int D, int BW, bool CLAMP>
__device__ __forceinline__ void pack4(uint8_t* row, int cl, uint32_t zq0, uint32_t zq1, uint32_t zq2, uint32_t zq3) {
    const uint32_t t = gather4<BW, CLAMP>(zq0, zq1, zq2, zq3);
    if constexpr (BW == 8) {
        *reinterpret_cast<uint32_t*>(row + 4 * cl) = t;
    } else if constexpr (BW == 4) {
        *reinterpret_cast<uint16_t*>(row + 2 * cl) = static_cast<uint16_t>(nibbles4(t));
    } else if constexpr (BW == 2) {
        row[cl] = static_cast<uint8_t>(crumbs4(t));
    } else {
        *reinterpret_cast<uint16_t*>(row + 2 * cl) = static_cast<uint16_t>(nibbles4(t));
        row[D / 2 + cl] = static_cast<uint8_t>(high_crumbs4(t));
    }
}

// Store 8 codes (CPL = 8 chunk) at width BW: one store per plane.
template <int D, int BW, bool CLAMP>
__device__ __forceinline__ void pack8(uint8_t* row, int cl, const uint32_t zq[8]) {
    const uint32_t t0 = gather4<BW, CLAMP>(zq[0], zq[1], zq[2], zq[3]);
    const uint32_t t1 = gather4<BW, CLAMP>(zq[4], zq[5], zq[6], zq[7]);
    if constexpr (BW == 8) {
        *reinterpret_cast<uint2*>(row + 8 * cl) = make_uint2(t0, t1);
    } else if constexpr (BW == 4) {
        *reinterpret_cast<uint32_t*>(row + 4 * cl) = __byte_perm(nibbles4(t0), nibbles4(t1), 0x5410);
    } else if constexpr (BW == 2) {
        *reinterpret_cast<uint16_t*>(row + 2 * cl) = static_cast<uint16_t>(__byte_perm(crumbs4(t0), crumbs4(t1), 0x0040));
    } else {
        *reinterpret_cast<uint32_t*>(row + 4 * cl) = __byte_perm(nibbles4(t0), nibbles4(t1), 0x5410);
        *reinterpret_cast<uint16_t*>(row + D / 2 + 2 * cl) =
            static_cast<uint16_t>(__byte_perm(high_crumbs4(t0), high_crumbs4(t1), 0x0040));
    }
}

// Runtime-width CPL = 4 forms (the state conversion kernels; one warp-uniform branch per row).
template <int D>
__device__ __forceinline__ void unpack4(const uint8_t* row, int cl, int b, float z[4]) {
    float2 a, c;
    switch (b) {
        case 8: unpack4<D, 8>(row, cl, a, c); break;
        case 4: unpack4<D, 4>(row, cl, a, c); break;
        case 2: unpack4<D, 2>(row, cl, a, c); break;
        case 16: {   // FP16 pivot row: the values themselves
            const uint2 u = *reinterpret_cast<const uint2*>(row + 8 * cl);
            a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
            c = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
            break;
        }
        default: unpack4<D, 6>(row, cl, a, c); break;
    }
    z[0] = a.x; z[1] = a.y; z[2] = c.x; z[3] = c.y;
}

// An FP16 pivot value: fp32 -> binary16, nearest-even, saturating at +-65504.
__device__ __forceinline__ __half pivot_half(float x) {
    return __float2half_rn(fminf(fmaxf(x, -kHalfMax), kHalfMax));
}

// Store 4 codes already limited to [-q_b, q_b].
template <int D>
__device__ __forceinline__ void pack4_store(uint8_t* row, int cl, int b, const int q[4]) {
    const uint32_t a = static_cast<uint32_t>(q[0]), bb = static_cast<uint32_t>(q[1]);
    const uint32_t c = static_cast<uint32_t>(q[2]), d = static_cast<uint32_t>(q[3]);
    switch (b) {
        case 8: pack4<D, 8, false>(row, cl, a, bb, c, d); break;
        case 4: pack4<D, 4, false>(row, cl, a, bb, c, d); break;
        case 2: pack4<D, 2, false>(row, cl, a, bb, c, d); break;
        default: pack4<D, 6, false>(row, cl, a, bb, c, d); break;
    }
}

// ------------------------------------------------------------------------------------------
// row reduction: every thread holds one partial per owned row (RPT values); the LPR lanes of
// a sub-row hold the partials of the same rows. Result: the full sum of row r lands in the
// lanes (s*LPR + hh*RPT + r) for hh in {0, 1}; returns it together with the row slot r.
// buf: per-warp scratch of 32 * (RPT + 1) floats (padded so both passes are conflict-free).
// ------------------------------------------------------------------------------------------

template <class M, typename T, typename Op>
__device__ __forceinline__ T row_reduce(T* buf, int lane, const T part[M::RPT], int& slot, Op op) {
    constexpr int RPT = M::RPT;
    constexpr int LPR = M::LPR;
    static_assert(LPR == 2 * RPT, "two lanes per row in the reduction");
#pragma unroll
    for (int r = 0; r < RPT; ++r) buf[lane * (RPT + 1) + r] = part[r];
    __syncwarp();
    const int s = lane / LPR, ll = lane % LPR;
    const int rr = ll % RPT, hh = ll / RPT;
    T acc = buf[(s * LPR + hh * RPT) * (RPT + 1) + rr];
#pragma unroll
    for (int m = 1; m < RPT; ++m) acc = op(acc, buf[(s * LPR + hh * RPT + m) * (RPT + 1) + rr]);
    acc = op(acc, __shfl_xor_sync(0xffffffffu, acc, RPT));
    __syncwarp();
    slot = rr;
    return acc;
}

struct OpAdd {
    template <typename T>
    __device__ T operator()(T x, T y) const { return x + y; }
};
struct OpMax {
    __device__ float operator()(float x, float y) const { return fmaxf(x, y); }
};

// Row (slot) of the value returned by row_reduce to this lane, and whether this lane is the
// one of the two holders that should act on it.
template <class M>
__device__ __forceinline__ int reduced_row(int warp, int lane, int slot, bool& owner) {
    owner = (lane % M::LPR) < M::RPT;
    return warp * M::kRowsPerWarp + slot * M::RPW + M::sub_row(lane);
}

// Byte offset of every row inside its tile (one warp): the integer rows first, in key order,
// then the FP16 pivot rows (width 16), in key order. Row i has D/8 * b_i bytes.
template <int D>
__device__ __forceinline__ int row_offsets_warp(const uint8_t* bits, uint16_t* roff, int lane) {
    constexpr int RL = D / 32;
    int loc[RL], sum_i = 0, sum_p = 0;
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        const int b = bits[lane * RL + r];
        loc[r] = b == 16 ? sum_p : sum_i;
        (b == 16 ? sum_p : sum_i) += b * (D / 8);
    }
    int inc_i = sum_i, inc_p = sum_p;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ti = __shfl_up_sync(0xffffffffu, inc_i, o);
        const int tp = __shfl_up_sync(0xffffffffu, inc_p, o);
        if (lane >= o) { inc_i += ti; inc_p += tp; }
    }
    const int total_i = __shfl_sync(0xffffffffu, inc_i, 31);
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        const int b = bits[lane * RL + r];
        const int base = b == 16 ? total_i + inc_p - sum_p : inc_i - sum_i;
        roff[lane * RL + r] = static_cast<uint16_t>(base + loc[r]);
    }
    return total_i + __shfl_sync(0xffffffffu, inc_p, 31);   // the tile's bytes
}

// Bit 2 of the device error word: a tile whose head-offset range cannot hold it (see below).
constexpr uint32_t kFlagBadLayout = 4u;

// Whether head h's byte range in a sequence, [head_off[h], end) with end = head_off[h+1] (or
// bytes_per_seq for the last head), can hold a tile of `tile_bytes` bytes: both ends 16-byte
// aligned, ascending, inside the sequence, and at least tile_bytes long. A kernel that gets false
// skips the tile (reads and writes nothing of it) and raises bit 2 of *flags, so a head-offset
// table that does not match the bit map, or a bytes_per_seq shorter than the table, never moves an
// access outside the tile's own range. tile_bytes < 0 checks the range alone (at most max_bytes).
__device__ __forceinline__ bool tile_range_ok(const int64_t* head_off, int H, int64_t bytes_per_seq, int h,
                                              int64_t tile_bytes, int64_t max_bytes, uint32_t* flags,
                                              int64_t* hoff_out = nullptr, int64_t* hend_out = nullptr) {
    const int64_t hoff = head_off[h];
    const int64_t hend = (h + 1 < H) ? head_off[h + 1] : bytes_per_seq;
    const int64_t need = tile_bytes >= 0 ? tile_bytes : 0;
    const bool ok = hoff >= 0 && ((hoff | hend) & 15) == 0 && hoff + need <= hend && hend <= bytes_per_seq &&
                    hend - hoff <= max_bytes;
    if (!ok && flags) atomicOr(flags, kFlagBadLayout);
    if (hoff_out) *hoff_out = hoff;
    if (hend_out) *hend_out = hend;
    return ok;
}

// Combine the per-thread column partials of the RPW sub-rows of a warp.
template <class M, typename T, typename Op, int N = 4>
__device__ __forceinline__ void combine_subrows(T v[N], Op op) {
#pragma unroll
    for (int m = M::LPR; m < 32; m <<= 1)
#pragma unroll
        for (int k = 0; k < N; ++k) v[k] = op(v[k], __shfl_xor_sync(0xffffffffu, v[k], m));
}

// ------------------------------------------------------------------------------------------
// bulk async copies (TMA engine, 1-D, no multicast) and mbarriers
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended for up to hint_ns while the phase is
// incomplete, so a waiting warp takes few issue slots from the warps that have work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Global -> shared bulk copy completing on `bar`. bytes: multiple of 16; both addresses
// 16-byte aligned.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Shared -> global bulk copy (1-D, TMA engine) in this thread's bulk-async group. bytes: a
// multiple of 16; both addresses 16-byte aligned. The writes of the shared source must be made
// visible to the async proxy first (fence_proxy_async_smem by each writing thread, then a barrier).
__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_addr(src_smem)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Until every committed bulk store of this thread has read its shared source (the buffer may be
// refilled) / has completed.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` for at most `limit_ns` nanoseconds of wall time. Returns
// false (and raises bit 0 of *flags, the caller's device error word) if the limit was reached.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                  uint32_t* flags) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 10000u)) return true;
        if (global_timer_ns() - t0 > limit_ns) break;
    }
    atomicOr(flags, 1u);
    return false;
}

}  // namespace stepq
