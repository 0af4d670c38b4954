// stepq_tile.cuh -- the register-tile mapping of a (sequence, head) state tile onto one CTA
// and the steps shared by the fused decode kernel and the tensor-core prefill chunk kernel:
// width-sorted row tables, column partial sums, and the refit and pack of the tile (the
// row factors of §4.3, the no-clip column start and the weighted least-squares column update
// of App. C.1, final codes packed per the state layout).
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

#include "stepq_device.cuh"

namespace stepq {

// Mapping of a tile onto one CTA: a thread owns 8 adjacent columns of RPT rows; LPR lanes span
// a row; a warp covers RPW rows per instruction and owns 16 consecutive slots (rows sorted by
// width).
template <int D>
struct DMap {
    static constexpr int kCols = 8;
    static constexpr int kThreads = (D == 128) ? 256 : 128;
    static constexpr int kMinBlocks = (D == 128) ? 2 : 4;
    static constexpr int kWarps = kThreads / 32;
    static constexpr int LPR = D / kCols;               // lanes per row
    static constexpr int RPW = 32 / LPR;                // rows per warp instruction
    static constexpr int RPT = D / (kWarps * RPW);      // rows per thread
    static constexpr int kRowsPerWarp = RPT * RPW;
    __device__ static int col_lane(int lane) { return lane % LPR; }
    __device__ static int sub_row(int lane) { return lane / LPR; }
    __device__ static int row(int warp, int lane, int r) { return warp * kRowsPerWarp + r * RPW + sub_row(lane); }
    // Row length of the column-partial buffers red[kWarps][2][kRedRow] of a kernel that finalises
    // columns with every thread: the two rows of a warp are 16 banks apart, so lanes 0-15 and
    // 16-31 of a warp reading the two rows at the same 16 columns are free of bank conflicts.
    static constexpr int kRedRow = D + 16;
    // The column such a thread finalises (16 per warp; lanes l and l + 16 share it), and which
    // of the two partial rows it sums.
    __device__ static int fin_col(int warp, int lane) { return 16 * warp + (lane & 15); }
    __device__ static int fin_row(int lane) { return lane >> 4; }
};

// The widths of a head's key rows lane*RL .. lane*RL + RL-1 (RL = D/32), one byte each.
template <int D>
__device__ __forceinline__ uint32_t head_widths(const uint8_t* bits_h, int lane) {
    if constexpr (D == 128) return *reinterpret_cast<const uint32_t*>(bits_h + 4 * lane);
    else return *reinterpret_cast<const uint16_t*>(bits_h + 2 * lane);
}

// One warp sorts the key rows of a head by bit width (stable). widths: head_widths() of the
// head's D widths. hmeta[slot] = row | width << 8 | byte offset << 16; hslot[row] = slot |
// width << 8. A width-16 row with kPiv false raises bit 1 of *flags.
template <int D, bool kPiv>
__device__ __forceinline__ int sort_head_rows_w(uint32_t widths, uint32_t* hmeta, uint16_t* hslot, int lane,
                                                uint32_t* flags) {
    // Width classes in slot order: 2, 4, 6, 8, then 16 (FP16 pivot rows). Byte offsets follow
    // the packed layout: integer rows in key order, then pivot rows in key order.
    constexpr int RL = D / 32, NC = 5;
    int bw[RL], loc[RL], rank[RL], sum_i = 0, sum_p = 0;
    int cnt[NC] = {0, 0, 0, 0, 0};
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        bw[r] = (widths >> (8 * r)) & 0xFF;
        const bool piv = bw[r] == 16;
        loc[r] = piv ? sum_p : sum_i;
        (piv ? sum_p : sum_i) += bw[r] * (D / 8);
        const int cls = piv ? 4 : (bw[r] >> 1) - 1;
        rank[r] = 0;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            if (c == cls) rank[r] = cnt[c];
            cnt[c] += (c == cls);
        }
    }
    int inc_i = sum_i, inc_p = sum_p;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ti = __shfl_up_sync(0xffffffffu, inc_i, o);
        const int tp = __shfl_up_sync(0xffffffffu, inc_p, o);
        if (lane >= o) { inc_i += ti; inc_p += tp; }
    }
    const int total_i = __shfl_sync(0xffffffffu, inc_i, 31);
    int excl_c[NC], base_c[NC], base = 0;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        int x = cnt[c];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        excl_c[c] = x - cnt[c];
        base_c[c] = base;
        base += __shfl_sync(0xffffffffu, x, 31);
    }
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        const int i = lane * RL + r;
        const bool piv = bw[r] == 16;
        const int cls = piv ? 4 : (bw[r] >> 1) - 1;
        int slot = 0;
#pragma unroll
        for (int c = 0; c < NC; ++c)
            if (c == cls) slot = base_c[c] + excl_c[c] + rank[r];
        int off = (piv ? total_i + inc_p - sum_p : inc_i - sum_i) + loc[r];
        int wb = bw[r];
        if (!kPiv && piv) {
            // A pivot row in a launch declared without pivots: flagged (bit 1); the row is
            // handled as an in-bounds 8-bit row so that nothing is read or written outside
            // the tile (its results are undefined).
            atomicOr(flags, 2u);
            wb = 8;
            off = min(off, D * D - D);
        }
        hmeta[slot] = static_cast<uint32_t>(i) | (static_cast<uint32_t>(wb) << 8) | (static_cast<uint32_t>(off) << 16);
        hslot[i] = static_cast<uint16_t>(slot | (wb << 8));
    }
    return total_i + __shfl_sync(0xffffffffu, inc_p, 31);   // the tile's bytes under this bit map
}

// As sort_head_rows_w, from the bit map row of the head (bits_h: D widths, 4-byte aligned).
template <int D, bool kPiv>
__device__ __forceinline__ int sort_head_rows(const uint8_t* bits_h, uint32_t* hmeta, uint16_t* hslot, int lane,
                                              uint32_t* flags) {
    return sort_head_rows_w<D, kPiv>(head_widths<D>(bits_h, lane), hmeta, hslot, lane, flags);
}

// The row widths that a per-row (mixed) code path handles: every width (kW = 0), or the widths
// of the bit mask kW (bit b for width b; width 16, the FP16 pivot rows, is governed by kPiv).
// The lowest declared width, the fallback, also takes the rows of any undeclared width.
template <int kW>
struct WidthSet {
    static constexpr bool has(int b) { return kW == 0 || ((kW >> b) & 1) != 0; }
    static constexpr int fallback =
        kW == 0 ? 2 : ((kW >> 2) & 1) ? 2 : ((kW >> 4) & 1) ? 4 : ((kW >> 6) & 1) ? 6 : 8;
    static constexpr bool tested(int b) { return has(b) && b != fallback; }   // its own branch
};

// Eight consecutive per-column values (columns 8cl .. 8cl+7) as four pairs.
__device__ __forceinline__ void load_cols8(const float* src, int cl, float2 out[4]) {
    const float4 a = *reinterpret_cast<const float4*>(src + 8 * cl);
    const float4 b = *reinterpret_cast<const float4*>(src + 8 * cl + 4);
    out[0] = make_float2(a.x, a.y);
    out[1] = make_float2(a.z, a.w);
    out[2] = make_float2(b.x, b.y);
    out[3] = make_float2(b.z, b.w);
}

// Sum (over the warp's sub-rows) the per-thread partials of eight columns and store them.
template <int D>
__device__ __forceinline__ void store_col_partials(float* dst, int lane, float2 v[4]) {
    using M = DMap<D>;
#pragma unroll
    for (int m = M::LPR; m < 32; m <<= 1)
#pragma unroll
        for (int p = 0; p < 4; ++p)
            v[p] = add2(v[p], make_float2(__shfl_xor_sync(0xffffffffu, v[p].x, m), __shfl_xor_sync(0xffffffffu, v[p].y, m)));
    if (lane < M::LPR) {
        const int cl = M::col_lane(lane);
        *reinterpret_cast<float4*>(dst + 8 * cl) = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
        *reinterpret_cast<float4*>(dst + 8 * cl + 4) = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
    }
}

// ---- phase 6: final codes, packed and stored ------------------------------------------------
// Codes are always limited to [-q_b, q_b]: the least-squares column scale is below the no-clip
// scale in most columns, so the limit is nearly always needed somewhere in a tile.
template <int D, int BW>
__device__ __forceinline__ void phase6_row(uint8_t* out, uint32_t mt, int cl, const float2 x[4], const float2 f[4]) {
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);
    uint32_t zq[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 t = fma2(x[p], f[p], M2);
        zq[2 * p] = __float_as_uint(t.x);
        zq[2 * p + 1] = __float_as_uint(t.y);
    }
    pack8<D, BW, true>(out + (mt >> 16), cl, zq);
}

// An FP16 pivot row: X_ij = xi_ij c_j (xi = alpha_i Y_ij for pivot rows), rounded to binary16
// (nearest-even, saturating) and stored straight to global memory.
template <int D>
__device__ __forceinline__ void phase6_pivot_row(uint8_t* out, uint32_t mt, int cl, const float2 x[4], const float2 cc[4]) {
    uint32_t h[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 v = mul2(x[p], cc[p]);
        __half2 hv = __halves2half2(pivot_half(v.x), pivot_half(v.y));
        h[p] = *reinterpret_cast<uint32_t*>(&hv);
    }
    *reinterpret_cast<uint4*>(out + (mt >> 16) + 16 * cl) = make_uint4(h[0], h[1], h[2], h[3]);
}

template <int D, int BW>
__device__ __forceinline__ void phase6_uniform(const uint32_t* meta, uint8_t* out, int warp, int lane,
                                               const float2 Z[][4], const float2 f[4], const float* colc) {
    using M = DMap<D>;
    const int cl = M::col_lane(lane);
    float2 cc[4];
    if constexpr (BW == 16) load_cols8(colc, cl, cc);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        if constexpr (BW == 16) phase6_pivot_row<D>(out, meta[M::row(warp, lane, r)], cl, Z[r], cc);
        else phase6_row<D, BW>(out, meta[M::row(warp, lane, r)], cl, Z[r], f);
    }
}

template <int D, bool kPiv, int kW = 0>
__device__ __forceinline__ void phase6_mixed(const uint32_t* meta, uint8_t* out, int warp, int lane,
                                             const float2 Z[][4], const float2 f[4], const float* colc) {
    using M = DMap<D>;
    using WS = WidthSet<kW>;
    const int cl = M::col_lane(lane);
    float2 cc[4] = {};
    if constexpr (kPiv) load_cols8(colc, cl, cc);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const uint32_t mt = meta[M::row(warp, lane, r)];
        const int bw = (mt >> 8) & 0xFF;
        if constexpr (WS::tested(8)) if (bw == 8) { phase6_row<D, 8>(out, mt, cl, Z[r], f); continue; }
        if constexpr (WS::tested(6)) if (bw == 6) { phase6_row<D, 6>(out, mt, cl, Z[r], f); continue; }
        if constexpr (WS::tested(4)) if (bw == 4) { phase6_row<D, 4>(out, mt, cl, Z[r], f); continue; }
        if constexpr (WS::tested(2)) if (bw == 2) { phase6_row<D, 2>(out, mt, cl, Z[r], f); continue; }
        if constexpr (kPiv) if (bw == 16) { phase6_pivot_row<D>(out, mt, cl, Z[r], cc); continue; }
        phase6_row<D, WS::fallback>(out, mt, cl, Z[r], f);
    }
}

// kPiv: the pivot-capable instantiation (width-16 rows handled); without it the code is leaner.
template <int D, bool kPiv, int kW = 0>
__device__ __forceinline__ void phase6(const uint32_t* meta, uint8_t* out, int warp, int lane, int ww,
                                       const float2 Z[][4], const float2 f[4], const float* colc) {
    switch (ww) {
        case 8: phase6_uniform<D, 8>(meta, out, warp, lane, Z, f, colc); break;
        case 6: phase6_uniform<D, 6>(meta, out, warp, lane, Z, f, colc); break;
        case 4: phase6_uniform<D, 4>(meta, out, warp, lane, Z, f, colc); break;
        case 2: phase6_uniform<D, 2>(meta, out, warp, lane, Z, f, colc); break;
        default:
            if constexpr (kPiv) {
                if (ww == 16) {
                    phase6_uniform<D, 16>(meta, out, warp, lane, Z, f, colc);
                    break;
                }
            }
            phase6_mixed<D, kPiv, kW>(meta, out, warp, lane, Z, f, colc);
            break;
    }
}

// ---- phases 3-6: row factors, no-clip column start, least-squares column update, final codes
// packed and stored. The tile is in registers as X_ij = alpha_i c_j Y_ij (Y in Z, alpha_i in
// sm.ak[kb][slot].z, c_j in sm.colc); with kUpdate the last token's rank-1 update
// Y += (k_i/alpha_i)(u_j/c_j) (k/alpha in sm.ak[kb][slot].xy, u/c in sm.colb) is applied first.
// r_out and c_out point at the scales of tile `tile`, out at the tile's packed bytes.
template <int D, bool kPiv, bool kUpdate, int kW = 0, class Sm>
__device__ __forceinline__ void refit_pack(Sm& sm, const uint32_t* meta, float2 (&Z)[DMap<D>::RPT][4], int ww, int kb,
                                           int tile, uint16_t* r_out, uint16_t* c_out, uint8_t* out) {
    using M = DMap<D>;
    constexpr int RPT = M::RPT;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);
    {
        float2 cf[4], ut[4];
        load_cols8(sm.colc, cl, cf);
        if constexpr (kUpdate) load_cols8(sm.colb, cl, ut);
        float part[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            float2 ka = make_float2(0.f, 0.f);
            if constexpr (kUpdate) {
                const float4 c = sm.ak[kb][M::row(warp, lane, r)];
                ka = make_float2(c.x, c.y);
            }
            float acc = 0.f;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                if constexpr (kUpdate) Z[r][p] = fma2(ka, ut[p], Z[r][p]);
                acc = fmaf(fabsf(Z[r][p].x), cf[p].x, acc);
                acc = fmaf(fabsf(Z[r][p].y), cf[p].y, acc);
            }
            part[r] = acc;
        }
        int slot;
        bool owner;
        const float rsum = row_reduce<M, float>(sm.rowbuf[warp], lane, part, slot, OpAdd());
        const int sl = reduced_row<M>(warp, lane, slot, owner);   // a slot index
        if (owner) {
            const uint32_t mt = meta[sl];
            const int i = mt & 0xFF, bw = (mt >> 8) & 0xFF;
            const float2 w2 = sm.wsl[sl];
            const float alpha = sm.ak[kb][sl].z;
            const __half rh = scale_to_half(fmaxf(alpha * rsum * (1.0f / D), kHalfMinNormal) * w2.y);
            r_out[static_cast<int64_t>(tile) * D + i] = __half_as_ushort(rh);
            const float rs = __half2float(rh) * znorm_of(bw);
            if (kPiv && bw == 16) {   // FP16 pivot row: xi = alpha Y, outside the shared column fit
                sm.rq[sl] = make_float4(alpha, alpha, 0.f, 0.f);
                sm.riq[sl] = 0.f;
            } else {
                const float e = alpha * rcp_approx(rs);
                const float g = w2.x * rs;
                sm.rq[sl] = make_float4(e, e, g * g, g * g);
                sm.riq[sl] = inv_qmax_of(bw);
            }
        }
        __syncwarp();
    }

    // ---- phase 4: xi = X / (c_j r~_i 2^(8-b_i)); column no-clip scale c0 -----------
    {
        float2 cmax[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) cmax[p] = make_float2(0.f, 0.f);
        if (ww != 0) {
#pragma unroll
            for (int r = 0; r < RPT; r += 2) {
                const float4 q4 = sm.rq[M::row(warp, lane, r)];
                const float4 q5 = sm.rq[M::row(warp, lane, r + 1)];
                const float2 e2 = make_float2(q4.x, q4.y), e3 = make_float2(q5.x, q5.y);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    Z[r][p] = mul2(Z[r][p], e2);
                    Z[r + 1][p] = mul2(Z[r + 1][p], e3);
                    cmax[p].x = max_abs3(cmax[p].x, Z[r][p].x, Z[r + 1][p].x);
                    cmax[p].y = max_abs3(cmax[p].y, Z[r][p].y, Z[r + 1][p].y);
                }
            }
            const float iq = sm.riq[warp * M::kRowsPerWarp];
#pragma unroll
            for (int p = 0; p < 4; ++p) cmax[p] = mul2(cmax[p], make_float2(iq, iq));
        } else {
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int sl = M::row(warp, lane, r);
                const float4 q4 = sm.rq[sl];
                const float2 e2 = make_float2(q4.x, q4.y);
                const float iq = sm.riq[sl];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    Z[r][p] = mul2(Z[r][p], e2);
                    cmax[p].x = fmaxf(cmax[p].x, fabsf(Z[r][p].x) * iq);
                    cmax[p].y = fmaxf(cmax[p].y, fabsf(Z[r][p].y) * iq);
                }
            }
        }
#pragma unroll
        for (int m = M::LPR; m < 32; m <<= 1)
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                cmax[p].x = fmaxf(cmax[p].x, __shfl_xor_sync(0xffffffffu, cmax[p].x, m));
                cmax[p].y = fmaxf(cmax[p].y, __shfl_xor_sync(0xffffffffu, cmax[p].y, m));
            }
        if (lane < M::LPR) {
            *reinterpret_cast<float4*>(&sm.red[warp][0][8 * cl]) = make_float4(cmax[0].x, cmax[0].y, cmax[1].x, cmax[1].y);
            *reinterpret_cast<float4*>(&sm.red[warp][0][8 * cl + 4]) = make_float4(cmax[2].x, cmax[2].y, cmax[3].x, cmax[3].y);
        }
    }
    __syncthreads();
    if (tid < D) {
        const int j = tid;
        float cm = 0.f;
#pragma unroll
        for (int w = 0; w < M::kWarps; ++w) cm = fmaxf(cm, sm.red[w][0][j]);
        const float cj = sm.colc[j];
        const float c0 = fmaxf(cj * cm, kHalfMinNormal);
        sm.col0[j] = c0;
        sm.colb[j] = cj * rcp_approx(c0);
    }
    __syncthreads();

    // ---- phase 5: codes at (r~, c0); weighted least-squares column update ----------
    {
        float2 f[4];
        load_cols8(sm.colb, cl, f);
        const float2 mM2 = make_float2(-kRoundMagic, -kRoundMagic);
        float2 num[4], den[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) num[p] = den[p] = make_float2(0.f, 0.f);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float4 q4 = sm.rq[M::row(warp, lane, r)];
            const float2 G2 = make_float2(q4.z, q4.w);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 z0 = add2(fma2(Z[r][p], f[p], M2), mM2);
                const float2 gz = mul2(G2, z0);
                num[p] = fma2(gz, Z[r][p], num[p]);
                den[p] = fma2(gz, z0, den[p]);
            }
        }
        store_col_partials<D>(sm.red[warp][0], lane, num);
        store_col_partials<D>(sm.red[warp][1], lane, den);
    }
    __syncthreads();
    if (tid < D) {
        const int j = tid;
        float ns = 0.f, ds = 0.f;
#pragma unroll
        for (int w = 0; w < M::kWarps; ++w) {
            ns += sm.red[w][0][j];
            ds += sm.red[w][1][j];
        }
        const float cj = sm.colc[j];
        const float c1 = ds > 0.f ? (cj * ns) * rcp_approx(ds) : sm.col0[j];
        const __half ch = scale_to_half(c1);
        c_out[static_cast<int64_t>(tile) * D + j] = __half_as_ushort(ch);
        sm.colb[j] = cj * rcp_approx(__half2float(ch));
    }
    __syncthreads();

    // ---- phase 6: final codes at (r~, c~), packed and stored -----------------------
    {
        float2 f[4];
        load_cols8(sm.colb, cl, f);
        phase6<D, kPiv, kW>(meta, out, warp, lane, ww, Z, f, sm.colc);
    }
}

}  // namespace stepq
