// stepq_prefill_wy.cu -- the prefill chunk (STEPQuant App. F.1 and App. B.2: reconstruct the
// packed state once, run the native chunk update over the chunk's tokens, refit and pack the
// boundary state once) in the chunked WY/UT form of the gated Delta rule, on the fifth-generation
// tensor cores of sm_100a.
//
// Per (sequence, head) tile with state S0 (d_k x d_v, d = 128) and C <= 64 tokens, gates g_t,
// gamma_t = g_1 ... g_t and R_ts = gamma_t / gamma_s, the recurrence of §2.1
//   S_t = g_t S_{t-1} + k_t u_t^T,   u_t = beta_t (v_t - g_t S_{t-1}^T k_t),   o_t = S_t^T q_t
// unrolls to S_t = gamma_t S0 + sum_{s<=t} R_ts k_s u_s^T, so that the rows u_t solve the unit
// lower triangular system (I + L) U = diag(beta) (V - diag(gamma) K S0) with
// L_ts = beta_t R_ts k_t.k_s (s < t). With T = (I + L)^-1:
//   U   = T diag(beta) V - T diag(beta gamma) K S0
//   O   = diag(gamma) Q S0 + (R o tril(Q K^T)) U
//   S_C = gamma_C S0 + (diag(gamma_C / gamma) K)^T U.
// Every product is an M = 128 tcgen05.mma (bf16 operands, fp32 accumulation in tensor memory).
// One operand of each product is exact in bf16: q, k and v are bf16 inputs and S0 enters as its
// integer codes Z (S0 = diag(r 2^(8-b)) Z diag(c), |Z| <= 127). The other operand, computed in
// fp32, is split into bf16 parts whose products are accumulated: three parts (high, middle, low:
// 24 significant bits, as fp32) for every product that reaches the boundary state, whose codes
// must agree with a float64 evaluation; two parts (about 2^-17) for the readout's P U, which takes
// the three largest of its four part products. T comes from a blocked inversion (16 x 16
// diagonal blocks by substitution, then block rows) on the CUDA cores. The boundary state then
// runs through the same refit and pack as the fused decode step (steps 4-6 of Table C2).
//
// Channel gates (one gate per key channel, D_t = diag(g_t), as in Kimi Delta Attention): with
// lambda_ti the running log2 of channel i's gate product and R_tsi = prod_{s < tau <= t} g_tau,i,
// the same rearrangement holds with the gate factors inside the channel sums:
//   L_ts = beta_t sum_i k_ti k_si R_tsi,   P_ts = sum_i q_ti k_si R_tsi (s <= t),
//   U    = T diag(beta) V - T diag(beta) (K o 2^lambda) S0,
//   O    = (Q o 2^lambda) S0 + P U,
//   S_C  = diag(2^lambda_C) S0 + (K o 2^(lambda_C - lambda))^T U.
// L and P are formed on the CUDA cores in fp32 through a hierarchy of reference tokens: the pairs
// whose token indices first differ in bit l are the (upper half, lower half) pairs of the aligned
// blocks of 2^(l+1) tokens, and with the last token of the lower half as reference R_tsi is the
// product of a factor of t (the gates from the upper half's start to t) and a factor of s (the
// gates after s to the lower half's end), both at most 1: no partial product can overflow,
// whatever the gates. The gate-scaled operands (K o 2^lambda, Q o 2^lambda, K o 2^(lambda_C -
// lambda)) are not exact in bf16, so both operands of W = T diag(beta) (K o 2^lambda) and of the
// boundary-state product are split in three parts, of which the six largest part products are
// accumulated (the three largest leave about 0.5 % of 8-bit column scales off those of a float64
// evaluation; six leave none, in a NumPy emulation of this arithmetic).
//
// One CTA per SM (the operands of a tile take 224 KB of shared memory), 256 threads, 512 TMEM
// columns; tiles are dealt round-robin. With one CTA of 8 warps per SM the phases' code must
// stay small: loops whose bodies are large are kept rolled (instruction-cache misses were the
// first stall reason when they were unrolled). The next tile's packed codes are copied by the bulk-copy
// engine while the current tile is computed; q, k and v arrive through 16-byte asynchronous
// copies straight into the tensor cores' operand layout.
#include <cuda_runtime.h>

#include "stepq_device.cuh"
#include "stepq_internal.h"
#include "stepq_tile.cuh"
#include "stepq_umma.cuh"

namespace stepq {
namespace {

constexpr int D = 128;        // d_k = d_v
constexpr int C = 64;         // tokens per tile pass (a shorter chunk is padded: k = q = v = 0,
                              // beta = 0, g = 1 leave every result unchanged)
constexpr int NT = 256;       // threads per CTA
using M = DMap<D>;
static_assert(M::kThreads == NT, "the refit runs on the decode kernel's thread mapping");

struct WyArgs {
    int B, H, num_tiles, chunk;
    const uint16_t* q;        // [chunk][B][H][D] bf16
    const uint16_t* k;
    const uint16_t* v;
    const float* beta;        // [chunk][B][H]
    const float* gate;        // [chunk][B][H]
    const uint8_t* bits;
    const float* w;
    const int64_t* head_off;
    int64_t bytes_per_seq;
    const uint8_t* packed_in;
    const uint16_t* r_in;
    const uint16_t* c_in;
    uint8_t* packed_out;
    uint16_t* r_out;
    uint16_t* c_out;
    float* o;                 // [chunk][B][H][D]
    uint32_t* flags;          // device error word (bit 0: a bounded wait gave up)
};

// Per-slot and per-column work space of the refit (same fields as the decode kernel's).
struct FitScratch {
    alignas(16) float4 ak[1][D];
    alignas(16) float4 rq[D];
    alignas(16) float2 wsl[D];
    alignas(16) float riq[D];
    alignas(16) float colc[D];
    alignas(16) float colb[D];
    alignas(16) float col0[D];
    alignas(16) float icol[D];
    alignas(16) float red[M::kWarps][2][D];
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
};

struct Small {
    alignas(16) uint32_t hmeta[D];   // per slot: row | width << 8 | byte offset << 16
    alignas(16) uint16_t hslot[D];   // per row: slot | width << 8
    alignas(16) float rho[D];        // r_i 2^(8 - b_i)
    alignas(16) float cs[D];         // c_j
    alignas(16) float icol[D];       // 1 / c_j
    alignas(16) float beta[C];
    alignas(16) float l2g[C];        // log2 gamma_t (a zero gate counts as 2^-64)
    alignas(16) float lamC[D];       // channel gates: lambda_C,i, the chunk's log2 gate product
    alignas(16) float lcarry[D];     // channel gates: lambda of the first 32 tokens (scan carry)
    alignas(8) uint64_t bar_mma;
    alignas(8) uint64_t bar_sc;      // the last round's boundary-state product, committed apart
    alignas(8) uint64_t bar_codes;
    uint32_t tmem;
    int tile_ok;                     // the tile's head range holds it under the bit map
    uint32_t pmask;                  // FP16 pivot rows: bit n set if rows 16 n to 16 n + 15 hold one
};

// Shared-memory map (bytes). The work region is reused phase by phase.
constexpr uint32_t OFF_KQ = 0;            // bf16 [K; Q]: rows t (k) and 64 + t (q), K-major over d
constexpr uint32_t OFF_V = 32768;         // bf16 V: rows t, K-major over d
constexpr uint32_t OFF_Z = 49152;         // bf16 codes Z: rows i, K-major over j
constexpr uint32_t OFF_CODES = 81920;     // the tile's packed codes (bulk copy)
constexpr uint32_t OFF_W = 98304;         // 127 KB work region, laid out per phase (see the kernel)
constexpr uint32_t OFF_SMALL = OFF_W + 127 * 1024;
constexpr int GLD = D + 4;                // padded row (floats) of the [token][channel] fp32 arrays
constexpr int PLD = C + 4;                // padded row (floats) of P
constexpr uint32_t SMEM_BYTES = OFF_SMALL + sizeof(Small);
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
static_assert(65536 + sizeof(FitScratch) <= OFF_SMALL - OFF_W, "refit work space");

// TMEM columns (512 allocated): G = [K;Q] K^T | W, later S_C | U_v | [W S0; gamma Q S0 + P U/c]
// | channel gates: lambda. Under channel gates G holds no product: its lanes 0-63 keep lambda_ti
// of channels i < 64 (lane t, column i) and its lanes 64-127 keep P (lane 64 + t, column s); the
// lambda columns' lanes 64-127 keep lambda_ti of channels i >= 64 (lane 64 + t, column i - 64).
constexpr uint32_t TM_G = 0, TM_W = 64, TM_U = 192, TM_S = 320, TM_LAM = 448;

constexpr uint64_t kWaitLimitNs = 2000000000ull;

// The six largest products of two operands each split in three bf16 parts (high, middle, low):
// part kPartA[n] of the first with part kPartB[n] of the second.
__device__ constexpr int kPartA[6] = {0, 0, 1, 0, 2, 1};
__device__ constexpr int kPartB[6] = {0, 1, 0, 2, 0, 1};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

// Eight fp32 values -> high bf16 parts and low bf16 parts (x - hi), each as one 16-byte chunk.
__device__ __forceinline__ void split8(const float x[8], uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * p], x[2 * p + 1]);
        const float2 hf = __bfloat1622float2(hb);
        h[p] = *reinterpret_cast<const uint32_t*>(&hb);
        l[p] = bf16x2_bits(x[2 * p] - hf.x, x[2 * p + 1] - hf.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Eight fp32 values -> three bf16 parts (x = hi + mid + lo to 24 significant bits).
__device__ __forceinline__ void split8x3(const float x[8], uint4& hi, uint4& mid, uint4& lo) {
    uint32_t h[4], m[4], l[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * p], x[2 * p + 1]);
        const float2 hf = __bfloat1622float2(hb);
        const float r0 = x[2 * p] - hf.x, r1 = x[2 * p + 1] - hf.y;
        const __nv_bfloat162 mb = __floats2bfloat162_rn(r0, r1);
        const float2 mf = __bfloat1622float2(mb);
        h[p] = *reinterpret_cast<const uint32_t*>(&hb);
        m[p] = *reinterpret_cast<const uint32_t*>(&mb);
        l[p] = bf16x2_bits(r0 - mf.x, r1 - mf.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    mid = make_uint4(m[0], m[1], m[2], m[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// fp32 64 x 64 matrices (L, T) with the 16-byte chunks of a row rotated by the row index.
__device__ __forceinline__ int sw64(int row, int col) {
    return row * 64 + ((((col >> 2) ^ row) & 15) << 2) + (col & 3);
}
// fp32 128 x 128 boundary state X, chunks rotated by row % 8.
__device__ __forceinline__ int swx(int row, int col) {
    return row * D + ((((col >> 2) ^ row) & 7) | ((col >> 2) & ~7)) * 4 + (col & 3);
}

// 2^x with the special function unit (relative error about 2^-22). The running log2 of the gate
// product is formed with the accurate log2f: its error would accumulate over the chunk.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float4 ld4(const float* m, int row, int col) {
    return *reinterpret_cast<const float4*>(m + sw64(row, col));
}
__device__ __forceinline__ float4 fma4(float a, float4 b, float4 c) {
    return make_float4(fmaf(a, b.x, c.x), fmaf(a, b.y, c.y), fmaf(a, b.z, c.z), fmaf(a, b.w, c.w));
}

// TMEM columns of this warp's lanes.
__device__ __forceinline__ uint32_t tm_at(uint32_t tm, int warp, uint32_t col) {
    return umma::tmem_at(tm, 32 * (warp & 3), static_cast<int>(col));
}

// ---- FP16 pivot rows --------------------------------------------------------------------------

// Eight stored binary16 values v_ij, j0 <= j < j0 + 8, of pivot row i (read from the packed input;
// zeros when the tile's head range failed its check).
__device__ __forceinline__ void pivot_values(const WyArgs& a, const Small& sm, int64_t tile_base, int i, int j0,
                                             float (&v)[8]) {
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (sm.tile_ok) {
        const uint8_t* row = a.packed_in + tile_base + (sm.hmeta[sm.hslot[i] & 0xFF] >> 16);
        raw = *reinterpret_cast<const uint4*>(row + 2 * j0);
    }
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        v[2 * p] = half_bits_to_float(static_cast<uint16_t>(w[p] & 0xFFFFu));
        v[2 * p + 1] = half_bits_to_float(static_cast<uint16_t>(w[p] >> 16));
    }
}

// v_ij / c_j (as v_ij times the reciprocal of c_j), the pivot row's entries of Z.
__device__ __forceinline__ void pivot_over_c(const WyArgs& a, const Small& sm, int64_t tile_base, int i, int j0,
                                             float (&x)[8]) {
    pivot_values(a, sm, tile_base, i, j0, x);
#pragma unroll
    for (int p = 0; p < 8; ++p) x[p] *= sm.icol[j0 + p];
}

// 4 KB slot n (n < 16) for the middle or low parts of one 16-row group of pivot rows, over
// regions free while the state product runs: Q (read by then), V (consumed by the second round),
// the codes buffer (the next tile's codes are fetched after this round) and the work region's top.
__device__ __forceinline__ uint16_t* zpart_slot(int n, uint16_t* KQ, uint16_t* Vs, uint8_t* codes, uint8_t* W) {
    if (n < 4) return KQ + 64 * D + 2048 * n;
    if (n < 8) return Vs + 2048 * (n - 4);
    if (n < 12) return reinterpret_cast<uint16_t*>(codes) + 2048 * (n - 8);
    return reinterpret_cast<uint16_t*>(W + 96 * 1024) + 2048 * (n - 12);
}

// ---- channel gates -------------------------------------------------------------------------

// TMEM column of lambda_ti for the 32 channels from i0 (a multiple of 32): channels 0-63 in
// lanes 0-63 (lane t) of the G columns, channels 64-127 in lanes 64-127 (lane 64 + t) of the
// lambda columns, so that every warp reaches the channels of its lane quarter.
__host__ __device__ constexpr uint32_t lam_col(int i0) {
    return i0 < 64 ? TM_G + static_cast<uint32_t>(i0) : TM_LAM + static_cast<uint32_t>(i0 - 64);
}
// The 32 channels whose lambda this warp's lane quarter holds (its token is 32 (warp & 1) + lane).
__device__ __forceinline__ int lam_channels(int warp) { return (warp & 2 ? 64 : 0) + 32 * (warp >> 2); }

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }

// One level of the reference hierarchy: the operands SK (every token) and SQ (upper halves only,
// compacted) of the pairs whose token indices first differ in bit LV. Thread (i, hh) holds the
// gates gv and the packed bf16 k | q << 16 of channel i, tokens 32 hh to 32 hh + 31.
//   upper half token t: factor = gates from the half's first token to t
//   lower half token s: factor = gates after s to the half's last token (1 for the last)
template <int LV>
__device__ __forceinline__ void level_operands(const float (&gv)[32], const uint32_t (&kq)[32], int hh, int i,
                                               float* SK, float* SQ) {
    constexpr int h = 1 << LV;
    float f = 1.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const bool up = LV == 5 ? hh != 0 : (j & h) != 0;
        const bool start = LV == 5 ? j == 0 : (j & (h - 1)) == 0;
        f = start ? gv[j] : f * gv[j];
        if (up) {
            const int t = 32 * hh + j;
            SK[t * GLD + i] = __uint_as_float(kq[j] << 16) * f;
            SQ[(((t >> (LV + 1)) << LV) | (t & (h - 1))) * GLD + i] = __uint_as_float(kq[j] & 0xFFFF0000u) * f;
        }
    }
    float b = 1.0f;
#pragma unroll
    for (int j = 31; j >= 0; --j) {
        const bool up = LV == 5 ? hh != 0 : (j & h) != 0;
        const bool end = LV == 5 ? j == 31 : (j & (h - 1)) == h - 1;
        if (end) b = 1.0f;
        if (!up) SK[(32 * hh + j) * GLD + i] = __uint_as_float(kq[j] << 16) * b;
        b *= gv[j];
    }
}

// Butterfly over the CS lanes of a tile (consecutive lanes, CS a power of two): each step halves
// the N values a lane holds, keeping the half its lane bit selects and adding the partner's copy
// of it; once one value is left the remaining steps add it up.
template <int NO, int CS, int O = 1, int N = NO>
__device__ __forceinline__ void reduce_tile(float (&v)[NO], int c) {
    if constexpr (O < CS) {
        if constexpr (N > 1) {
            const bool up = (c & O) != 0;
#pragma unroll
            for (int j = 0; j < N / 2; ++j) {
                const float send = up ? v[j] : v[j + N / 2];
                const float keep = up ? v[j + N / 2] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, O);
            }
            reduce_tile<NO, CS, 2 * O, N / 2>(v, c);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
            reduce_tile<NO, CS, 2 * O, 1>(v, c);
        }
    }
}

// The pair products of level LV: for t in the upper and s in the lower half of each aligned block
// of 2^(LV+1) tokens, L_ts = beta_t sum_i SK_ti SK_si (into the sw64 layout) and
// P_ts = sum_i SQ_t'i SK_si (into Pf). Pairs are dealt in TT x TT tiles, the 128 channels of a tile
// split over CS consecutive lanes (strided by 4 CS floats, so the lanes of a tile read adjacent
// 16-byte chunks), and the CS partial sums folded by reduce_tile.
template <int LV>
__device__ __forceinline__ void level_pairs(const float* SK, const float* SQ, const float* beta, float* Lf, float* Pf,
                                            int tid) {
    constexpr int h = 1 << LV;
    constexpr int TT = LV >= 2 ? 4 : (LV == 1 ? 2 : 1);
    constexpr int NB = h / TT;                      // t- (and s-) tile rows per half
    constexpr int NTILE = (32 / h) * NB * NB;
    constexpr int CS = NT / NTILE;
    constexpr int NG = D / (4 * CS);                // float4 channel groups per lane
    constexpr int NO = 2 * TT * TT;                 // L then P outputs of a tile
    static_assert(CS >= 1 && CS <= 32 && NG >= 1, "level tiling");
    const int tile = tid / CS, c = tid % CS;
    const int seg = tile / (NB * NB), rr = tile % (NB * NB);
    const int tb = rr / NB, sb = rr % NB;
    const int t0 = 2 * h * seg + h + TT * tb, s0 = 2 * h * seg + TT * sb, q0 = h * seg + TT * tb;
    float v[NO];
#pragma unroll
    for (int e = 0; e < NO; ++e) v[e] = 0.0f;
#pragma unroll 2
    for (int g = 0; g < NG; ++g) {
        const int i = 4 * c + 4 * CS * g;
        float4 kt[TT], qt[TT], ks[TT];
#pragma unroll
        for (int a = 0; a < TT; ++a) {
            kt[a] = *reinterpret_cast<const float4*>(SK + (t0 + a) * GLD + i);
            qt[a] = *reinterpret_cast<const float4*>(SQ + (q0 + a) * GLD + i);
            ks[a] = *reinterpret_cast<const float4*>(SK + (s0 + a) * GLD + i);
        }
#pragma unroll
        for (int a = 0; a < TT; ++a)
#pragma unroll
            for (int b = 0; b < TT; ++b) {
                float& l = v[a * TT + b];
                float& p = v[TT * TT + a * TT + b];
                l = fmaf(kt[a].x, ks[b].x, l); l = fmaf(kt[a].y, ks[b].y, l);
                l = fmaf(kt[a].z, ks[b].z, l); l = fmaf(kt[a].w, ks[b].w, l);
                p = fmaf(qt[a].x, ks[b].x, p); p = fmaf(qt[a].y, ks[b].y, p);
                p = fmaf(qt[a].z, ks[b].z, p); p = fmaf(qt[a].w, ks[b].w, p);
            }
    }
    reduce_tile<NO, CS>(v, c);
    constexpr int HS = ilog2(CS) < ilog2(NO) ? ilog2(CS) : ilog2(NO);   // halving steps taken
    constexpr int NF = NO >> HS;                                         // values left per lane
    if ((c >> HS) == 0) {
        int base = 0;
#pragma unroll
        for (int k = 0; k < HS; ++k) base += ((c >> k) & 1) * (NO >> (k + 1));
#pragma unroll
        for (int j = 0; j < NF; ++j) {
            const int e = base + j, f = e % (TT * TT);
            const int t = t0 + f / TT, s = s0 + f % TT;
            if (e < TT * TT)
                Lf[sw64(t, s)] = beta[t] * v[j];
            else
                Pf[t * PLD + s] = v[j];
        }
    }
}

// The gates of a tile's tokens t < chunk into Gs (fp32 [token][channel], rows of GLD floats);
// rows past the chunk are left as they are (the scans take them as 1).
__device__ __forceinline__ void load_gates(const WyArgs& a, int tile, int tid, float* Gs) {
    const int64_t T = a.num_tiles;
#pragma unroll 1
    for (int m = 0; m < 8; ++m) {
        const int e = tid + NT * m;                  // 64 rows x 32 chunks of 16 bytes
        const int row = e >> 5, ch = e & 31;
        if (row < a.chunk) cp_async16(Gs + row * GLD + 4 * ch, a.gate + (static_cast<int64_t>(row) * T + tile) * D + 4 * ch, 16u);
    }
    cp_async_commit();
}

// The small inputs of a tile, loaded into registers one tile ahead: warp 0 the gates and betas
// of tokens 2 lane and 2 lane + 1, warp 1 the head's row widths, threads < 128 r_i and c_i.
struct Ahead {
    float g0, g1, b0, b1;
    uint32_t widths;
    uint32_t rc;          // r_i | c_i << 16 (binary16 bits)
    int64_t codes_src;    // thread 0: the packed codes of the tile after this one (their copy is
    uint32_t codes_bytes; // queued while this one is computed); 0 bytes if its head range is bad
    bool has_next;        // thread 0: there is a tile after this one
};

template <bool kChan>
__device__ __forceinline__ Ahead load_ahead(const WyArgs& a, int tile, int tid, int warp, int lane) {
    Ahead n{1.0f, 1.0f, 0.0f, 0.0f, 0u, 0u, 0, 0u, false};
    const int64_t T = a.num_tiles;
    if (tid == 0 && tile + static_cast<int>(gridDim.x) < a.num_tiles) {
        const int t2 = tile + gridDim.x, b2 = t2 / a.H, h2 = t2 % a.H;
        int64_t hoff, hend;
        n.has_next = true;
        if (tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h2, -1, 2 * D * D, a.flags, &hoff, &hend)) {
            n.codes_src = static_cast<int64_t>(b2) * a.bytes_per_seq + hoff;
            n.codes_bytes = static_cast<uint32_t>(min(hend - hoff, static_cast<int64_t>(D) * D));
        }
    }
    if (warp == 0) {
        const int t0 = 2 * lane, t1 = t0 + 1;
        if (t0 < a.chunk) {
            if (!kChan) n.g0 = __ldg(a.gate + t0 * T + tile);
            n.b0 = __ldg(a.beta + t0 * T + tile);
        }
        if (t1 < a.chunk) {
            if (!kChan) n.g1 = __ldg(a.gate + t1 * T + tile);
            n.b1 = __ldg(a.beta + t1 * T + tile);
        }
    } else if (warp == 1) {
        n.widths = head_widths<D>(a.bits + static_cast<int64_t>(tile % a.H) * D, lane);
    }
    if (tid < D)
        n.rc = static_cast<uint32_t>(__ldg(a.r_in + static_cast<int64_t>(tile) * D + tid)) |
               static_cast<uint32_t>(__ldg(a.c_in + static_cast<int64_t>(tile) * D + tid)) << 16;
    return n;
}

// q, k, v rows t < chunk (zero rows past it) of a tile into the K-major operand layout.
__device__ __forceinline__ void load_tokens(const WyArgs& a, int tile, int tid, uint16_t* KQ, uint16_t* Vs) {
    const int64_t T = a.num_tiles;
#pragma unroll 1
    for (int m = 0; m < 12; ++m) {
        const int e = tid + NT * m;              // 3 matrices x 64 rows x 16 chunks
        const int mat = e >> 10, row = (e & 7) | ((e >> 7) & 7) << 3, ch = (e >> 3) & 15;
        const uint16_t* src = mat == 0 ? a.k : (mat == 1 ? a.q : a.v);
        const bool valid = row < a.chunk;
        src += (static_cast<int64_t>(valid ? row : 0) * T + tile) * D + 8 * ch;
        uint16_t* dst = mat == 2 ? Vs + umma::kmajor_off(row, 8 * ch, D) : KQ + umma::kmajor_off(row + 64 * mat, 8 * ch, D);
        cp_async16(dst, src, valid ? 16u : 0u);
    }
    cp_async_commit();
}

// Queues the copy of a tile's packed codes; a head range that cannot hold a tile copies nothing
// (the arrival still completes the barrier phase, and the tile is skipped where it is computed).
__device__ __forceinline__ void issue_codes(const WyArgs& a, int tile, uint8_t* dst, uint64_t* bar) {
    const int b = tile / a.H, h = tile % a.H;
    int64_t hoff, hend;
    const bool ok = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, -1, 2 * D * D, a.flags, &hoff, &hend);
    const uint32_t bytes = ok ? static_cast<uint32_t>(min(hend - hoff, static_cast<int64_t>(D) * D)) : 0u;
    mbar_arrive_expect_tx(bar, bytes);
    if (bytes) bulk_load(dst, a.packed_in + static_cast<int64_t>(b) * a.bytes_per_seq + hoff, bytes, bar);
}

template <bool kChan, bool kPiv>
__global__ void __launch_bounds__(NT, 1) prefill_wy_kernel(const WyArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    Small& sm = *reinterpret_cast<Small*>(smem + OFF_SMALL);
    uint16_t* KQ = reinterpret_cast<uint16_t*>(smem + OFF_KQ);
    uint16_t* Vs = reinterpret_cast<uint16_t*>(smem + OFF_V);
    uint16_t* Zs = reinterpret_cast<uint16_t*>(smem + OFF_Z);
    uint8_t* codes = smem + OFF_CODES;
    // The work region, phase by phase (KB offsets):
    //   B: [T''; T'] planes 0, 16, 32 | L 64 | T 80 | G blocks 96
    //   C: [W rho; gamma Q rho] planes 0, 32, 64
    //   D: U/c planes 0, 16 | U~ planes 32, 48, 64 | P planes 88, 96 (their MMA operand starts
    //      8 KB earlier: rows 0-63 there only reach TMEM lanes already consumed)
    //   E: X 0 | refit work space 64
    // Under channel gates, before B: gates, then lambda, then SK 0 | SQ 34 | L 64 | P 104; in B the
    // (K o 2^lambda) planes at 48, 64 and 102 (L and the G blocks are consumed by then).
    uint8_t* W = smem + OFF_W;
    auto h16 = [&](uint32_t kb) { return reinterpret_cast<uint16_t*>(W + 1024 * kb); };
    uint16_t* AT[3] = {h16(0), h16(16), h16(32)};
    float* Lf = reinterpret_cast<float*>(W + 64 * 1024);
    float* Tf = reinterpret_cast<float*>(W + 80 * 1024);
    float* Gt = reinterpret_cast<float*>(W + 96 * 1024);
    uint16_t* WQ[3] = {h16(0), h16(32), h16(64)};
    uint16_t* BUC[2] = {h16(0), h16(16)};
    uint16_t* BUT[3] = {h16(32), h16(48), h16(64)};
    uint16_t* Pp[2] = {h16(88), h16(96)};
    float* X = reinterpret_cast<float*>(W);
    FitScratch& fit = *reinterpret_cast<FitScratch*>(W + 64 * 1024);
    float* Gs = reinterpret_cast<float*>(W);
    float* SK = reinterpret_cast<float*>(W);
    float* SQ = reinterpret_cast<float*>(W + 34 * 1024);
    float* Pf = reinterpret_cast<float*>(W + 104 * 1024);
    uint16_t* KT[3] = {h16(48), h16(64), h16(102)};

    if (tid == 0) {
        mbar_init(&sm.bar_mma, 1);
        mbar_init(&sm.bar_sc, 1);
        mbar_init(&sm.bar_codes, 1);
        fence_barrier_init();
    }
    if (warp == 0) umma::tmem_alloc(&sm.tmem, 512);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tm = sm.tmem;
    uint32_t mma_phase = 0, sc_phase = 0, codes_phase = 0;
    bool codes_pending = false;
    const int64_t T = a.num_tiles;

    // Waits for the tensor core's last commit; false (uniformly over the CTA) if it never came.
    auto wait_bar = [&](uint64_t* bar, uint32_t& phase) -> bool {
        const bool ok = mbar_wait_bounded(bar, phase, kWaitLimitNs, a.flags);
        phase ^= 1u;
        const bool all = !__syncthreads_or(!ok);
        umma::fence_after_sync();
        return all;
    };
    auto wait_mma = [&]() -> bool { return wait_bar(&sm.bar_mma, mma_phase); };
    // Orders this thread's shared-memory writes and TMEM reads before an MMA that the
    // issuing thread starts after the barrier.
    auto to_tensor_core = [&]() {
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
    };

    // The first tile's inputs; later tiles' arrive during the previous tile's refit.
    Ahead nx{};
    if (static_cast<int>(blockIdx.x) < a.num_tiles) {
        if (tid == 0) {
            issue_codes(a, blockIdx.x, codes, &sm.bar_codes);
            codes_pending = true;
        }
        load_tokens(a, blockIdx.x, tid, KQ, Vs);
        nx = load_ahead<kChan>(a, blockIdx.x, tid, warp, lane);
    }

    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
        const int b = tile / a.H, h = tile % a.H;
        const int64_t tile_base = static_cast<int64_t>(b) * a.bytes_per_seq + a.head_off[h];
        const int next = tile + gridDim.x;

        // ---- A: tables, gates, scales, codes -----------------------------------------------
        if constexpr (kChan) load_gates(a, tile, tid, Gs);
        if (warp == 1) {
            const int total = sort_head_rows_w<D, kPiv>(nx.widths, sm.hmeta, sm.hslot, lane, a.flags);
            // A head range that cannot hold the tile under the bit map: the tile is computed on
            // whatever the buffers hold and none of its results is written.
            if (lane == 0) sm.tile_ok = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, total, 2 * D * D, a.flags);
            if constexpr (kPiv) {   // the 16-row groups (key order) that hold FP16 pivot rows
                uint32_t m = 0;
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    if (((nx.widths >> (8 * r)) & 0xFFu) == 16u) m |= 1u << ((4 * lane + r) >> 4);
                m = __reduce_or_sync(0xffffffffu, m);
                if (lane == 0) sm.pmask = m;
            }
        }
        if (warp == 0) {   // beta and the running log2 of the gate product (a zero gate counts 2^-64)
            const float l0 = log2f(fmaxf(nx.g0, 0x1p-64f));
            const float l1 = l0 + log2f(fmaxf(nx.g1, 0x1p-64f));
            float inc = l1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            const float excl = inc - l1;
            sm.l2g[2 * lane] = excl + l0;
            sm.l2g[2 * lane + 1] = excl + l1;
            sm.beta[2 * lane] = nx.b0;
            sm.beta[2 * lane + 1] = nx.b1;
        }
        __syncthreads();
        float w_slot = 1.0f;   // row-impact factor of slot tid (used by the refit)
        if (tid < D) {
            const int bw = sm.hslot[tid] >> 8;
            const float cj = half_bits_to_float(static_cast<uint16_t>(nx.rc >> 16));
            // an FP16 pivot row enters as Z_ij = v_ij / c_j with rho_i = 1
            sm.rho[tid] = kPiv && bw == 16 ? 1.0f : half_bits_to_float(static_cast<uint16_t>(nx.rc & 0xFFFFu)) * znorm_of(bw);
            sm.cs[tid] = cj;
            sm.icol[tid] = 1.0f / cj;
            w_slot = __ldg(a.w + static_cast<int64_t>(h) * D + (sm.hmeta[tid] & 0xFF));
        }
        const bool ok = mbar_wait_bounded(&sm.bar_codes, codes_phase, kWaitLimitNs, a.flags);
        codes_phase ^= 1u;
        if (__syncthreads_or(!ok)) break;
        codes_pending = false;
#pragma unroll 1
        for (int m = 0; m < 8; ++m) {
            const int e = tid + NT * m;              // 128 rows x 16 chunks, 8 rows per 8 lanes
            const int i = (e & 7) | ((e >> 7) << 3), cc = (e >> 3) & 15;
            const uint32_t hs = sm.hslot[i];
            const uint8_t* row = codes + (sm.hmeta[hs & 0xFF] >> 16);
            float2 z[4];
            switch (hs >> 8) {
                case 8: unpack8<D, 8>(row, cc, z); break;
                case 6: unpack8<D, 6>(row, cc, z); break;
                case 4: unpack8<D, 4>(row, cc, z); break;
                case 16:
                    if constexpr (kPiv) {   // the high bf16 part of v_ij / c_j (values from global memory)
                        float x[8];
                        pivot_over_c(a, sm, tile_base, i, 8 * cc, x);
#pragma unroll
                        for (int p = 0; p < 4; ++p) z[p] = make_float2(x[2 * p], x[2 * p + 1]);
                        break;
                    }
                    [[fallthrough]];
                default: unpack8<D, 2>(row, cc, z); break;
            }
            *reinterpret_cast<uint4*>(Zs + umma::kmajor_off(i, 8 * cc, D)) =
                make_uint4(bf16x2_bits(z[0].x, z[0].y), bf16x2_bits(z[1].x, z[1].y), bf16x2_bits(z[2].x, z[2].y),
                           bf16x2_bits(z[3].x, z[3].y));
        }
        cp_async_wait_all();
        to_tensor_core();
        if (tid == 0) {
            umma::fence_after_sync();
            if (!kChan) {
                const uint32_t id = umma::idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma::mma_bf16(tm + TM_G, umma::desc_kmajor(KQ, ks, D), umma::desc_kmajor(KQ, ks, D), id, ks > 0);
                umma::commit(&sm.bar_mma);
            }
            if (!kPiv && nx.has_next) {   // the codes buffer is free: fetch the next tile's
                mbar_arrive_expect_tx(&sm.bar_codes, nx.codes_bytes);
                if (nx.codes_bytes) bulk_load(codes, a.packed_in + nx.codes_src, nx.codes_bytes, &sm.bar_codes);
                codes_pending = true;
            }
        }
        if constexpr (!kChan) {
            if (!wait_mma()) break;
        } else {
            // ---- A': lambda, and L and P through the reference hierarchy ---------------------
            const int i = tid & (D - 1), hh = tid >> 7;   // channel i, tokens 32 hh to 32 hh + 31
            float gv[32];
            uint32_t kq[32];
            float lam = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int t = 32 * hh + j;
                gv[j] = t < a.chunk ? Gs[t * GLD + i] : 1.0f;
                kq[j] = static_cast<uint32_t>(KQ[umma::kmajor_off(t, i, D)]) |
                        static_cast<uint32_t>(KQ[umma::kmajor_off(64 + t, i, D)]) << 16;
                lam += log2f(fmaxf(gv[j], 0x1p-64f));
                Gs[t * GLD + i] = lam;
            }
            if (hh == 0) sm.lcarry[i] = lam;
            __syncthreads();
            if (hh == 1) {
                const float carry = sm.lcarry[i];
#pragma unroll
                for (int j = 0; j < 32; ++j) Gs[(32 + j) * GLD + i] += carry;
                sm.lamC[i] = lam + carry;
            }
            __syncthreads();
            {   // lambda into TMEM, each warp the 32 channels of its lane quarter
                const int t = 32 * (warp & 1) + lane, i0 = lam_channels(warp);
                float v[32];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 x = *reinterpret_cast<const float4*>(Gs + t * GLD + i0 + 4 * q4);
                    v[4 * q4] = x.x; v[4 * q4 + 1] = x.y; v[4 * q4 + 2] = x.z; v[4 * q4 + 3] = x.w;
                }
                umma::tmem_st32(tm_at(tm, warp, lam_col(i0)), v);
            }
            umma::fence_before_sync();
            __syncthreads();
            level_operands<5>(gv, kq, hh, i, SK, SQ);
            __syncthreads();
            level_pairs<5>(SK, SQ, sm.beta, Lf, Pf, tid);
            __syncthreads();
            level_operands<4>(gv, kq, hh, i, SK, SQ);
            __syncthreads();
            level_pairs<4>(SK, SQ, sm.beta, Lf, Pf, tid);
            __syncthreads();
            level_operands<3>(gv, kq, hh, i, SK, SQ);
            __syncthreads();
            level_pairs<3>(SK, SQ, sm.beta, Lf, Pf, tid);
            __syncthreads();
            level_operands<2>(gv, kq, hh, i, SK, SQ);
            __syncthreads();
            level_pairs<2>(SK, SQ, sm.beta, Lf, Pf, tid);
            __syncthreads();
            level_operands<1>(gv, kq, hh, i, SK, SQ);
            __syncthreads();
            level_pairs<1>(SK, SQ, sm.beta, Lf, Pf, tid);
            __syncthreads();
            level_operands<0>(gv, kq, hh, i, SK, SQ);
            __syncthreads();
            level_pairs<0>(SK, SQ, sm.beta, Lf, Pf, tid);
            {   // P_tt = q_t.k_t; zeros on and above the diagonal of L's 16 x 16 diagonal blocks
                const int t = tid >> 2, cg = tid & 3;
                float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint4 kb = *reinterpret_cast<const uint4*>(KQ + umma::kmajor_off(t, 32 * cg + 8 * m, D));
                    const uint4 qb = *reinterpret_cast<const uint4*>(KQ + umma::kmajor_off(64 + t, 32 * cg + 8 * m, D));
                    const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w}, qw[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        acc0 = fmaf(__uint_as_float(qw[p] << 16), __uint_as_float(kw[p] << 16), acc0);
                        acc1 = fmaf(__uint_as_float(qw[p] & 0xFFFF0000u), __uint_as_float(kw[p] & 0xFFFF0000u), acc1);
                    }
                }
                float acc = acc0 + acc1;
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (cg == 0) Pf[t * PLD + t] = acc;
                const int blk = tid >> 6, r = (tid >> 2) & 15, c4 = 4 * (tid & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (c4 + e >= r) Lf[sw64(16 * blk + r, 16 * blk + c4 + e)] = 0.0f;
            }
            __syncthreads();
            if (warp & 2) {   // P into TMEM lanes 64-127 (lane 64 + t, column s)
                const int t = 32 * (warp & 1) + lane, hf = warp >> 2;
                float v[32];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 x = *reinterpret_cast<const float4*>(Pf + t * PLD + 32 * hf + 4 * q4);
                    v[4 * q4] = x.x; v[4 * q4 + 1] = x.y; v[4 * q4 + 2] = x.z; v[4 * q4 + 3] = x.w;
                }
                umma::tmem_st32(tm_at(tm, warp, TM_G + 32 * hf), v);
            }
            umma::fence_before_sync();
            __syncthreads();
            umma::fence_after_sync();
        }

        // ---- B: L, T = (I + L)^-1, and the [T diag(beta); T diag(beta gamma)] planes ---------
        if (warp < 2) {   // lanes 0-63: row t of K K^T (under channel gates L is already formed)
          if constexpr (!kChan) {
            const int t = tid;
            const float lt = sm.l2g[t], bt = sm.beta[t];
#pragma unroll 1
            for (int c32 = 0; c32 < 2; ++c32) {
                float g[32];
                umma::tmem_ld32(tm_at(tm, warp, TM_G + 32 * c32), g);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const int s0 = 32 * c32 + 4 * q4;
                    const float4 l2 = *reinterpret_cast<const float4*>(sm.l2g + s0);
                    const float ls[4] = {l2.x, l2.y, l2.z, l2.w};
                    float l[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) l[e] = s0 + e < t ? bt * ex2(lt - ls[e]) * g[4 * q4 + e] : 0.0f;
                    *reinterpret_cast<float4*>(Lf + sw64(t, s0)) = make_float4(l[0], l[1], l[2], l[3]);
                }
            }
          }
        } else {   // T above the diagonal blocks is zero
            for (int e = tid - 64; e < 6 * 64; e += NT - 64) {
                const int blk = e >> 6, rr = (e >> 2) & 15, cq = e & 3;
                const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                *reinterpret_cast<float4*>(Tf + sw64(16 * bi + rr, 16 * bj + 4 * cq)) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        umma::fence_before_sync();
        __syncthreads();
        if (tid < 64) {   // diagonal 16 x 16 blocks by substitution, one column per thread
            const int o = 16 * (tid >> 4), c = tid & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = r == c ? 1.0f : 0.0f;
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                float acc0 = 0.0f, acc1 = 0.0f;   // L_rr' = 0 for r' >= r
#pragma unroll
                for (int u4 = 0; u4 < (r + 3) / 4; ++u4) {
                    const float4 l = ld4(Lf, o + r, o + 4 * u4);
                    acc0 = fmaf(l.x, x[4 * u4], acc0);
                    acc1 = fmaf(l.y, x[4 * u4 + 1], acc1);
                    acc0 = fmaf(l.z, x[4 * u4 + 2], acc0);
                    acc1 = fmaf(l.w, x[4 * u4 + 3], acc1);
                }
                if (r > c) x[r] = -(acc0 + acc1);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tf[sw64(o + r, o + c)] = x[r];
        }
        __syncthreads();
        // Block rows: T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj = -sum_k G_ik T_kj with G_ik = T_ii L_ik,
        // formed once; then one level per distance lv = i - j. A thread computes four adjacent
        // entries of one 16 x 16 block.
#pragma unroll 1
        for (int e = tid; e < 6 * 64; e += NT) {
            const int pr = e >> 6, ra = (e >> 2) & 15, c4 = 4 * (e & 3);
            const int i = pr < 1 ? 1 : (pr < 3 ? 2 : 3), k = pr - i * (i - 1) / 2;
            float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u0 = 0; u0 < 16; u0 += 4) {
                const float4 t = ld4(Tf, 16 * i + ra, 16 * i + u0);
                g = fma4(t.x, ld4(Lf, 16 * i + u0, 16 * k + c4), g);
                g = fma4(t.y, ld4(Lf, 16 * i + u0 + 1, 16 * k + c4), g);
                g = fma4(t.z, ld4(Lf, 16 * i + u0 + 2, 16 * k + c4), g);
                g = fma4(t.w, ld4(Lf, 16 * i + u0 + 3, 16 * k + c4), g);
            }
            *reinterpret_cast<float4*>(Gt + (pr * 16 + ra) * 16 + c4) = g;
        }
        __syncthreads();
#pragma unroll 1
        for (int lv = 1; lv <= 3; ++lv) {
            if (tid < 64 * (4 - lv)) {
                const int j = tid >> 6, i = j + lv, ra = (tid >> 2) & 15, c4 = 4 * (tid & 3);
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
                for (int k = j; k < i; ++k) {
                    const float* gr = Gt + ((i * (i - 1) / 2 + k) * 16 + ra) * 16;
#pragma unroll
                    for (int u0 = 0; u0 < 16; u0 += 4) {
                        const float4 g = *reinterpret_cast<const float4*>(gr + u0);
                        acc = fma4(g.x, ld4(Tf, 16 * k + u0, 16 * j + c4), acc);
                        acc = fma4(g.y, ld4(Tf, 16 * k + u0 + 1, 16 * j + c4), acc);
                        acc = fma4(g.z, ld4(Tf, 16 * k + u0 + 2, 16 * j + c4), acc);
                        acc = fma4(g.w, ld4(Tf, 16 * k + u0 + 3, 16 * j + c4), acc);
                    }
                }
                *reinterpret_cast<float4*>(Tf + sw64(16 * i + ra, 16 * j + c4)) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
        }
        // [T''; T'] with T''_ts = T_ts beta_s (rows 0-63), T'_ts = T_ts beta_s gamma_s (rows 64-127).
#pragma unroll 1
        for (int m = 0; m < 4; ++m) {
            const int e = tid + NT * m;              // 128 rows x 8 chunks
            const int row = (e & 7) | ((e >> 6) << 3), cc = (e >> 3) & 7;
            const int t = row & 63, s0 = 8 * cc;
            const float4 t0 = ld4(Tf, t, s0), t1 = ld4(Tf, t, s0 + 4);
            const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            float x[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float f = row < 64 || kChan ? sm.beta[s0 + p] : sm.beta[s0 + p] * ex2(sm.l2g[s0 + p]);
                x[p] = tv[p] * f;
            }
            uint4 hi, mid, lo;
            split8x3(x, hi, mid, lo);
            *reinterpret_cast<uint4*>(AT[0] + umma::kmajor_off(row, s0, C)) = hi;
            *reinterpret_cast<uint4*>(AT[1] + umma::kmajor_off(row, s0, C)) = mid;
            *reinterpret_cast<uint4*>(AT[2] + umma::kmajor_off(row, s0, C)) = lo;
        }
        if constexpr (kChan) {   // the planes of K o 2^lambda (rows t, channels i), every warp 32 channels
            {
                const int t = 32 * (warp & 1) + lane;
                {
                    const int i0 = lam_channels(warp);
                    float lv[32];
                    umma::tmem_ld32(tm_at(tm, warp, lam_col(i0)), lv);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 kb = *reinterpret_cast<const uint4*>(KQ + umma::kmajor_off(t, i0 + 8 * q, D));
                        const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w};
                        float x[8];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            x[2 * p] = __uint_as_float(kw[p] << 16) * ex2(lv[8 * q + 2 * p]);
                            x[2 * p + 1] = __uint_as_float(kw[p] & 0xFFFF0000u) * ex2(lv[8 * q + 2 * p + 1]);
                        }
                        uint4 hi, mid, lo;
                        split8x3(x, hi, mid, lo);
                        *reinterpret_cast<uint4*>(KT[0] + umma::kmajor_off(t, i0 + 8 * q, D)) = hi;
                        *reinterpret_cast<uint4*>(KT[1] + umma::kmajor_off(t, i0 + 8 * q, D)) = mid;
                        *reinterpret_cast<uint4*>(KT[2] + umma::kmajor_off(t, i0 + 8 * q, D)) = lo;
                    }
                }
            }
        }
        to_tensor_core();
        if (tid == 0) {   // [T''; T'] K (W = T' K in lanes 64-127) and [T''; T'] V (U_v in lanes 0-63)
            umma::fence_after_sync();
            const uint32_t id = umma::idesc_bf16(128, 128, false, true);
            if constexpr (!kChan) {
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks) {
                        const uint64_t da = umma::desc_kmajor(AT[p], ks, C);
                        umma::mma_bf16(tm + TM_W, da, umma::desc_mnmajor(KQ, ks, D), id, p > 0 || ks > 0);
                        umma::mma_bf16(tm + TM_U, da, umma::desc_mnmajor(Vs, ks, D), id, p > 0 || ks > 0);
                    }
            } else {   // U_v from the three parts of T diag(beta); W from six part products with K o 2^lambda
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        umma::mma_bf16(tm + TM_U, umma::desc_kmajor(AT[p], ks, C), umma::desc_mnmajor(Vs, ks, D), id,
                                       p > 0 || ks > 0);
#pragma unroll
                for (int pq = 0; pq < 6; ++pq)
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        umma::mma_bf16(tm + TM_W, umma::desc_kmajor(AT[kPartA[pq]], ks, C),
                                       umma::desc_mnmajor(KT[kPartB[pq]], ks, D), id, pq > 0 || ks > 0);
            }
            umma::commit(&sm.bar_mma);
        }
        if (!wait_mma()) break;

        // ---- C: the [W diag(rho); diag(gamma) Q diag(rho)] planes ---------------------------
        {
            const int t = 32 * (warp & 1) + lane, hf = warp >> 2;
            if (warp & 2) {   // W rows from TMEM lanes 64 + t
#pragma unroll 1
                for (int c32 = 0; c32 < 2; ++c32) {
                    float wv[32];
                    umma::tmem_ld32(tm_at(tm, warp, TM_W + 64 * hf + 32 * c32), wv);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i0 = 64 * hf + 32 * c32 + 8 * q;
                        const float4 r0 = *reinterpret_cast<const float4*>(sm.rho + i0);
                        const float4 r1 = *reinterpret_cast<const float4*>(sm.rho + i0 + 4);
                        const float x[8] = {wv[8 * q] * r0.x, wv[8 * q + 1] * r0.y, wv[8 * q + 2] * r0.z,
                                            wv[8 * q + 3] * r0.w, wv[8 * q + 4] * r1.x, wv[8 * q + 5] * r1.y,
                                            wv[8 * q + 6] * r1.z, wv[8 * q + 7] * r1.w};
                        uint4 hi, mid, lo;
                        split8x3(x, hi, mid, lo);
                        *reinterpret_cast<uint4*>(WQ[0] + umma::kmajor_off(t, i0, D)) = hi;
                        *reinterpret_cast<uint4*>(WQ[1] + umma::kmajor_off(t, i0, D)) = mid;
                        *reinterpret_cast<uint4*>(WQ[2] + umma::kmajor_off(t, i0, D)) = lo;
                    }
                }
            } else if constexpr (!kChan) {   // gamma_t q_t rho
                const float gt = ex2(sm.l2g[t]);
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    const int i0 = 64 * hf + 8 * cc;
                    const uint4 qb = *reinterpret_cast<const uint4*>(KQ + umma::kmajor_off(64 + t, i0, D));
                    const uint32_t qw[4] = {qb.x, qb.y, qb.z, qb.w};
                    const float4 r0 = *reinterpret_cast<const float4*>(sm.rho + i0);
                    const float4 r1 = *reinterpret_cast<const float4*>(sm.rho + i0 + 4);
                    const float rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                    float x[8];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        x[2 * p] = __uint_as_float(qw[p] << 16) * gt * rr[2 * p];
                        x[2 * p + 1] = __uint_as_float(qw[p] & 0xFFFF0000u) * gt * rr[2 * p + 1];
                    }
                    uint4 hi, mid, lo;
                    split8x3(x, hi, mid, lo);
                    *reinterpret_cast<uint4*>(WQ[0] + umma::kmajor_off(64 + t, i0, D)) = hi;
                    *reinterpret_cast<uint4*>(WQ[1] + umma::kmajor_off(64 + t, i0, D)) = mid;
                    *reinterpret_cast<uint4*>(WQ[2] + umma::kmajor_off(64 + t, i0, D)) = lo;
                }
            }
            if constexpr (kChan) {   // 2^lambda_ti q_ti rho_i, every warp the 32 channels of its lane quarter
                const int ch0 = lam_channels(warp);
                float lv[32];
                umma::tmem_ld32(tm_at(tm, warp, lam_col(ch0)), lv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i0 = ch0 + 8 * q;
                    const uint4 qb = *reinterpret_cast<const uint4*>(KQ + umma::kmajor_off(64 + t, i0, D));
                    const uint32_t qw[4] = {qb.x, qb.y, qb.z, qb.w};
                    const float4 r0 = *reinterpret_cast<const float4*>(sm.rho + i0);
                    const float4 r1 = *reinterpret_cast<const float4*>(sm.rho + i0 + 4);
                    const float rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                    float x[8];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        x[2 * p] = __uint_as_float(qw[p] << 16) * ex2(lv[8 * q + 2 * p]) * rr[2 * p];
                        x[2 * p + 1] = __uint_as_float(qw[p] & 0xFFFF0000u) * ex2(lv[8 * q + 2 * p + 1]) * rr[2 * p + 1];
                    }
                    uint4 hi, mid, lo;
                    split8x3(x, hi, mid, lo);
                    *reinterpret_cast<uint4*>(WQ[0] + umma::kmajor_off(64 + t, i0, D)) = hi;
                    *reinterpret_cast<uint4*>(WQ[1] + umma::kmajor_off(64 + t, i0, D)) = mid;
                    *reinterpret_cast<uint4*>(WQ[2] + umma::kmajor_off(64 + t, i0, D)) = lo;
                }
            }
        }
        if constexpr (kPiv) {
            // The middle and low bf16 parts of v_ij / c_j (the high part is in Z) for every 16-row
            // group holding pivot rows, zero in its integer rows: slots 2n and 2n + 1 for the n-th
            // such group.
            __syncthreads();
            const uint32_t pm = sm.pmask;
            int n = 0;
#pragma unroll 1
            for (int ks = 0; ks < D / 16; ++ks) {
                if (!((pm >> ks) & 1u)) continue;
                const int i = 16 * ks + (tid >> 4), cc = tid & 15;
                uint4 hi, mid = make_uint4(0u, 0u, 0u, 0u), lo = make_uint4(0u, 0u, 0u, 0u);
                if ((sm.hslot[i] >> 8) == 16) {
                    float x[8];
                    pivot_over_c(a, sm, tile_base, i, 8 * cc, x);
                    split8x3(x, hi, mid, lo);
                }
                const int off = umma::kmajor_off(i, 8 * cc, D) - 2048 * ks;
                *reinterpret_cast<uint4*>(zpart_slot(2 * n, KQ, Vs, codes, W) + off) = mid;
                *reinterpret_cast<uint4*>(zpart_slot(2 * n + 1, KQ, Vs, codes, W) + off) = lo;
                ++n;
            }
        }
        to_tensor_core();
        if (tid == 0) {   // [W rho; gamma Q rho] Z: lanes 0-63 W S0, lanes 64-127 gamma Q S0 (without c)
            umma::fence_after_sync();
            const uint32_t id = umma::idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma::mma_bf16(tm + TM_S, umma::desc_kmajor(WQ[p], ks, D), umma::desc_mnmajor(Zs, ks, D), id,
                                   p > 0 || ks > 0);
            if constexpr (kPiv) {   // the pivot rows' lower parts: A high x Z middle, A middle x Z middle, A high x Z low
                const uint32_t pm = sm.pmask;
                int n = 0;
#pragma unroll 1
                for (int ks = 0; ks < D / 16; ++ks) {
                    if (!((pm >> ks) & 1u)) continue;
                    const uint64_t dm = umma::smem_desc(smem_addr(zpart_slot(2 * n, KQ, Vs, codes, W)), D * 16u, 128u);
                    const uint64_t dl = umma::smem_desc(smem_addr(zpart_slot(2 * n + 1, KQ, Vs, codes, W)), D * 16u, 128u);
                    umma::mma_bf16(tm + TM_S, umma::desc_kmajor(WQ[0], ks, D), dm, id, 1u);
                    umma::mma_bf16(tm + TM_S, umma::desc_kmajor(WQ[1], ks, D), dm, id, 1u);
                    umma::mma_bf16(tm + TM_S, umma::desc_kmajor(WQ[0], ks, D), dl, id, 1u);
                    ++n;
                }
            }
            umma::commit(&sm.bar_mma);
        }
        if (!wait_mma()) break;
        if constexpr (kPiv) {   // the pivot parts' slots are consumed: fetch the next tile's codes
            if (tid == 0 && nx.has_next) {
                mbar_arrive_expect_tx(&sm.bar_codes, nx.codes_bytes);
                if (nx.codes_bytes) bulk_load(codes, a.packed_in + nx.codes_src, nx.codes_bytes, &sm.bar_codes);
                codes_pending = true;
            }
        }

        // ---- D: U = U_v - (W S0) diag(c); the U/c and U~ planes; the P planes ---------------
        {
            const int t = 32 * (warp & 1) + lane, hf = warp >> 2;
            if (!(warp & 2)) {   // TMEM lanes t: U_v and W S0
                const float ratio = kChan ? 1.0f : ex2(sm.l2g[C - 1] - sm.l2g[t]);
#pragma unroll 1
                for (int c16 = 0; c16 < 4; ++c16) {
                    float uv[16], ws[16];
                    umma::tmem_ld16x2(tm_at(tm, warp, TM_U + 64 * hf + 16 * c16), tm_at(tm, warp, TM_S + 64 * hf + 16 * c16),
                                      uv, ws);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int j0 = 64 * hf + 16 * c16 + 8 * half;
                        float xc[8], xt[8];
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            const float u = fmaf(-sm.cs[j0 + p], ws[8 * half + p], uv[8 * half + p]);
                            xc[p] = u * sm.icol[j0 + p];
                            xt[p] = u * ratio;
                        }
                        uint4 hi, lo;
                        split8(xc, hi, lo);
                        *reinterpret_cast<uint4*>(BUC[0] + umma::kmajor_off(t, j0, D)) = hi;
                        *reinterpret_cast<uint4*>(BUC[1] + umma::kmajor_off(t, j0, D)) = lo;
                        uint4 mid;
                        split8x3(xt, hi, mid, lo);
                        *reinterpret_cast<uint4*>(BUT[0] + umma::kmajor_off(t, j0, D)) = hi;
                        *reinterpret_cast<uint4*>(BUT[1] + umma::kmajor_off(t, j0, D)) = mid;
                        *reinterpret_cast<uint4*>(BUT[2] + umma::kmajor_off(t, j0, D)) = lo;
                    }
                }
            } else {             // TMEM lanes 64 + t: Q K^T row t -> P row t, s in [32 hf, 32 hf + 32)
                const float lt = sm.l2g[t];
                float g[32];
                umma::tmem_ld32(tm_at(tm, warp, TM_G + 32 * hf), g);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int s0 = 32 * hf + 8 * q;
                    float x[8];
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        x[p] = s0 + p <= t ? (kChan ? g[8 * q + p] : ex2(lt - sm.l2g[s0 + p]) * g[8 * q + p]) : 0.0f;
                    uint4 hi, lo;
                    split8(x, hi, lo);
                    *reinterpret_cast<uint4*>(Pp[0] + umma::kmajor_off(t, s0, C)) = hi;
                    *reinterpret_cast<uint4*>(Pp[1] + umma::kmajor_off(t, s0, C)) = lo;
                }
            }
            if constexpr (kChan) {   // the planes of K o 2^(lambda_C - lambda) over K, Q and V (consumed)
                {
                    uint16_t* KH[3] = {KQ, KQ + 64 * D, Vs};
                    {
                        const int i0 = lam_channels(warp);
                        float lv[32];
                        umma::tmem_ld32(tm_at(tm, warp, lam_col(i0)), lv);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int off = umma::kmajor_off(t, i0 + 8 * q, D);
                            const uint4 kb = *reinterpret_cast<const uint4*>(KQ + off);
                            const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w};
                            const float4 c0 = *reinterpret_cast<const float4*>(sm.lamC + i0 + 8 * q);
                            const float4 c1 = *reinterpret_cast<const float4*>(sm.lamC + i0 + 8 * q + 4);
                            const float lc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                            float x[8];
#pragma unroll
                            for (int p = 0; p < 4; ++p) {
                                x[2 * p] = __uint_as_float(kw[p] << 16) * ex2(lc[2 * p] - lv[8 * q + 2 * p]);
                                x[2 * p + 1] = __uint_as_float(kw[p] & 0xFFFF0000u) * ex2(lc[2 * p + 1] - lv[8 * q + 2 * p + 1]);
                            }
                            uint4 hi, mid, lo;
                            split8x3(x, hi, mid, lo);
                            *reinterpret_cast<uint4*>(KH[0] + off) = hi;
                            *reinterpret_cast<uint4*>(KH[1] + off) = mid;
                            *reinterpret_cast<uint4*>(KH[2] + off) = lo;
                        }
                    }
                }
            }
        }
        to_tensor_core();
        if (tid == 0) {
            umma::fence_after_sync();
            // O: lanes 64-127 of TM_S += P (U/c), three part products. The A operand's rows 0-63
            // are the 8 KB before each P plane; they only add to lanes 0-63, already consumed.
            const uint32_t id_o = umma::idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int pq = 0; pq < 3; ++pq) {
                const int p = pq == 2 ? 1 : 0, q = pq == 1 ? 1 : 0;
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    umma::mma_bf16(tm + TM_S, umma::desc_kmajor(Pp[p] - 64 * C, ks, C), umma::desc_mnmajor(BUC[q], ks, D),
                                   id_o, 1u);
            }
            umma::commit(&sm.bar_mma);   // the readouts can be written while S_C is computed
            // S_C - gamma_C S0 = K^T U~ into the W columns (W was consumed in C).
            const uint32_t id_s = umma::idesc_bf16(128, 128, true, true);
            if constexpr (!kChan) {
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        umma::mma_bf16(tm + TM_W, umma::desc_mnmajor(KQ, ks, D), umma::desc_mnmajor(BUT[p], ks, D), id_s,
                                       p > 0 || ks > 0);
            } else {   // (K o 2^(lambda_C - lambda))^T U: six part products
                const uint16_t* KH[3] = {KQ, KQ + 64 * D, Vs};
#pragma unroll
                for (int pq = 0; pq < 6; ++pq)
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        umma::mma_bf16(tm + TM_W, umma::desc_mnmajor(KH[kPartA[pq]], ks, D),
                                       umma::desc_mnmajor(BUT[kPartB[pq]], ks, D), id_s, pq > 0 || ks > 0);
            }
            umma::commit(&sm.bar_sc);
        }
        if (!wait_mma()) break;

        // ---- E: readouts, the boundary state X, its refit and pack --------------------------
        {
            const int hf = warp >> 2;
            if (warp & 2) {   // o_t = c (gamma Q S0 + P U/c), TMEM lanes 64 + t
                const int t = 32 * (warp & 1) + lane;
                float* orow = a.o + (static_cast<int64_t>(t) * T + tile) * D;
#pragma unroll 1
                for (int c32 = 0; c32 < 2; ++c32) {
                    float ov[32];
                    umma::tmem_ld32(tm_at(tm, warp, TM_S + 64 * hf + 32 * c32), ov);
                    if (t < a.chunk && sm.tile_ok) {
                        const int j0 = 64 * hf + 32 * c32;
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 cj = *reinterpret_cast<const float4*>(sm.cs + j0 + 4 * q4);
                            *reinterpret_cast<float4*>(orow + j0 + 4 * q4) =
                                make_float4(cj.x * ov[4 * q4], cj.y * ov[4 * q4 + 1], cj.z * ov[4 * q4 + 2], cj.w * ov[4 * q4 + 3]);
                        }
                    }
                }
            }
            // X_ij = (K^T U~)_ij + gamma_C rho_i c_j Z_ij, TMEM lane i, columns j in [64 hf, 64 hf + 64).
            if (!wait_bar(&sm.bar_sc, sc_phase)) break;
            const int i = 32 * (warp & 3) + lane;
            const float fi = (kChan ? ex2(sm.lamC[i]) : ex2(sm.l2g[C - 1])) * sm.rho[i];
#pragma unroll 1
            for (int c32 = 0; c32 < 2; ++c32) {
                float sv[32];
                umma::tmem_ld32(tm_at(tm, warp, TM_W + 64 * hf + 32 * c32), sv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j0 = 64 * hf + 32 * c32 + 8 * q;
                    const uint4 zb = *reinterpret_cast<const uint4*>(Zs + umma::kmajor_off(i, j0, D));
                    const uint32_t zw[4] = {zb.x, zb.y, zb.z, zb.w};
                    const float4 c0 = *reinterpret_cast<const float4*>(sm.cs + j0);
                    const float4 c1 = *reinterpret_cast<const float4*>(sm.cs + j0 + 4);
                    const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    float x[8];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        x[2 * p] = fmaf(fi * cc[2 * p], __uint_as_float(zw[p] << 16), sv[8 * q + 2 * p]);
                        x[2 * p + 1] = fmaf(fi * cc[2 * p + 1], __uint_as_float(zw[p] & 0xFFFF0000u), sv[8 * q + 2 * p + 1]);
                    }
                    if constexpr (kPiv) {
                        if ((sm.hslot[i] >> 8) == 16) {   // pivot row: gamma_C v_ij from the stored binary16 values
                            float v[8];
                            pivot_values(a, sm, tile_base, i, j0, v);
#pragma unroll
                            for (int p = 0; p < 8; ++p) x[p] = fmaf(fi, v[p], sv[8 * q + p]);
                        }
                    }
                    *reinterpret_cast<float4*>(X + swx(i, j0)) = make_float4(x[0], x[1], x[2], x[3]);
                    *reinterpret_cast<float4*>(X + swx(i, j0 + 4)) = make_float4(x[4], x[5], x[6], x[7]);
                }
            }
            if (tid < D) {   // the refit's constants: alpha = 1 and c = 1 (X is explicit)
                fit.wsl[tid] = make_float2(w_slot, rcp_approx(w_slot));
                fit.ak[0][tid] = make_float4(0.0f, 0.0f, 1.0f, 1.0f);
                fit.colc[tid] = 1.0f;
            }
        }
        umma::fence_before_sync();
        __syncthreads();
        if (next < a.num_tiles) {   // the next tile's q, k, v and small inputs arrive during the refit
            load_tokens(a, next, tid, KQ, Vs);
            nx = load_ahead<kChan>(a, next, tid, warp, lane);
        }
        {
            float2 Zr[M::RPT][4];
            const int cl = M::col_lane(lane);
#pragma unroll
            for (int r = 0; r < M::RPT; ++r) {
                const int row = sm.hmeta[M::row(warp, lane, r)] & 0xFF;
                const float4 x0 = *reinterpret_cast<const float4*>(X + swx(row, 8 * cl));
                const float4 x1 = *reinterpret_cast<const float4*>(X + swx(row, 8 * cl + 4));
                Zr[r][0] = make_float2(x0.x, x0.y);
                Zr[r][1] = make_float2(x0.z, x0.w);
                Zr[r][2] = make_float2(x1.x, x1.y);
                Zr[r][3] = make_float2(x1.z, x1.w);
            }
            const int w0 = (sm.hmeta[warp * M::kRowsPerWarp] >> 8) & 0xFF;
            const int w1 = (sm.hmeta[warp * M::kRowsPerWarp + M::kRowsPerWarp - 1] >> 8) & 0xFF;
            const int ww = (w0 == w1) ? w0 : 0;
            if (sm.tile_ok)   // uniform over the CTA
                refit_pack<D, kPiv, false>(fit, sm.hmeta, Zr, ww, 0, tile, a.r_out, a.c_out, a.packed_out + tile_base);
        }
        __syncthreads();   // the next tile rewrites the tables and the regions
    }

    // Copies still in flight (a wait above gave up) are waited for, boundedly, before exit.
    cp_async_wait_all();
    if (tid == 0 && codes_pending) mbar_wait_bounded(&sm.bar_codes, codes_phase, kWaitLimitNs, a.flags);
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_free(tm, 512);
}

}  // namespace
}  // namespace stepq

using namespace stepq;

extern "C" int stepq_prefill_chunk_wy(stepq_dims dims, int chunk, const uint16_t* q, const uint16_t* k,
                                      const uint16_t* v, const float* beta, const float* gate, const uint8_t* bits,
                                      const float* w, const int64_t* head_off, int64_t bytes_per_seq,
                                      const uint8_t* packed_in, const uint16_t* r_in, const uint16_t* c_in,
                                      uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out, float* o, void* stream) {
    const char* fn = "stepq_prefill_chunk_wy";
    clear_error();
    int rc = check_dims(dims, fn);
    if (rc) return rc;
    if (chunk < 1) return set_error(STEPQ_EINVAL, "%s: chunk=%d", fn, chunk);
    if (dims.dk != D || chunk > C)
        return set_error(STEPQ_EUNSUPPORTED,
                         "%s: the tensor-core chunk form needs d = 128 and at most %d tokens (d=%d chunk=%d)", fn, C,
                         dims.dk, chunk);
    if (dims.B == 0) return STEPQ_OK;
    rc = check_ptrs(fn, {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate}, {"bits", bits}, {"w", w},
                         {"head_off", head_off}, {"packed_in", packed_in}, {"r_in", r_in}, {"c_in", c_in},
                         {"packed_out", packed_out}, {"r_out", r_out}, {"c_out", c_out}, {"o", o}});
    if (rc) return rc;
    if (bytes_per_seq <= 0 || (bytes_per_seq & 15))
        return set_error(STEPQ_EINVAL, "%s: bytes_per_seq=%lld", fn, (long long)bytes_per_seq);
    const long long tiles = static_cast<long long>(dims.B) * dims.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "%s: too many tiles", fn);
    uint32_t* flags = nullptr;
    rc = device_flags_ptr(&flags);
    if (rc) return rc;
    WyArgs a{dims.B, dims.H, static_cast<int>(tiles), chunk, q, k, v, beta, gate, bits, w, head_off, bytes_per_seq,
             packed_in, r_in, c_in, packed_out, r_out, c_out, o, flags};
    const bool chan = dims.gate_per_channel != 0, piv = dims.pivots != 0;
    const void* kernel = chan ? (piv ? reinterpret_cast<const void*>(&prefill_wy_kernel<true, true>)
                                     : reinterpret_cast<const void*>(&prefill_wy_kernel<true, false>))
                              : (piv ? reinterpret_cast<const void*>(&prefill_wy_kernel<false, true>)
                                     : reinterpret_cast<const void*>(&prefill_wy_kernel<false, false>));
    int grid = 0;
    rc = persistent_grid(kernel, NT, SMEM_BYTES, tiles, fn, &grid);
    if (rc) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (chan && piv) prefill_wy_kernel<true, true><<<grid, NT, SMEM_BYTES, st>>>(a);
    else if (chan) prefill_wy_kernel<true, false><<<grid, NT, SMEM_BYTES, st>>>(a);
    else if (piv) prefill_wy_kernel<false, true><<<grid, NT, SMEM_BYTES, st>>>(a);
    else prefill_wy_kernel<false, false><<<grid, NT, SMEM_BYTES, st>>>(a);
    return check_launch(fn);
}

extern "C" int stepq_prefill_chunk(stepq_dims dims, int chunk, const uint16_t* q, const uint16_t* k,
                                   const uint16_t* v, const float* beta, const float* gate, const uint8_t* bits,
                                   const float* w, const int64_t* head_off, int64_t bytes_per_seq,
                                   const uint8_t* packed_in, const uint16_t* r_in, const uint16_t* c_in,
                                   uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out, float* o, void* stream) {
    // The tensor-core form under scalar gates; under channel gates its gate-weighted pair
    // products on the CUDA cores make it slower than the sequential form (KDA workload, 64-token
    // chunk: 3.04 against 2.90 ms), so the sequential form is taken there.
    const bool wy = dims.dk == 128 && dims.dv == 128 && dims.gate_per_channel == 0 && chunk >= 1 &&
                    chunk <= STEPQ_WY_MAX_CHUNK;
    return (wy ? stepq_prefill_chunk_wy : stepq_prefill_chunk_seq)(dims, chunk, q, k, v, beta, gate, bits, w, head_off,
                                                                   bytes_per_seq, packed_in, r_in, c_in, packed_out,
                                                                   r_out, c_out, o, stream);
}
