// stepq_decode.cu -- the fused quantized decode step (STEPQuant, Table C2) for sm_100a.
//
// One persistent CTA per SM slot walks over (sequence, head) tiles. For each tile the bulk-copy
// (TMA) engine stages the packed codes, the old scales, q/k/v, the gate and the head's bit map
// and row-impact vector into shared memory, double buffered so that the next tile's copy runs
// while this one is computed. The tile then lives in registers (a thread owns 4 columns of 16
// rows) through every phase:
//   1 unpack + dequantise (the column scale is factored out: Xi_ij = X_ij / c_j), and the two
//     column dot products k^T D S and q^T D S of the Delta rule;
//   2 u = beta (v - k^T D S), o = q^T X = q^T D S + (q.k) u          (§2.1, Table C2 step 3);
//   3 X = D S + k u^T and the row factors m_i = mean_j |X_ij|        (§4.3 "Row factors");
//   4 the no-clip column initialisation c0_j                         (fit start);
//   5 codes at (r, c0) and the weighted least-squares column update   (App. C.1);
//   6 final codes at (r, c), packed and stored straight to HBM.
// Rows are visited sorted by bit width, so almost every warp runs a width-specialised unpack
// and pack; floating-point work runs on packed f32x2 instructions. Column reductions cross
// warps through shared memory, row reductions stay inside a warp. The state is read once and
// written once; no tensor cores (a rank-1 update per token is not a dense contraction).
#include <cuda_runtime.h>

#include "stepq_device.cuh"
#include "stepq_internal.h"

namespace stepq {

// Device error word: bit 0 = a bounded wait for a tile copy gave up.
__device__ uint32_t g_stepq_flags = 0;

struct DecodeArgs {
    int B, H, gate_per_channel, num_tiles;
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* beta;
    const float* gate;
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
    float* o;
};

template <int D>
struct DecodeSmem {
    using M = Map<D>;
    struct Stage {
        alignas(16) uint8_t codes[D * D];   // room for an all-8-bit tile
        alignas(16) uint16_t r[D];
        alignas(16) uint16_t c[D];
        alignas(16) uint16_t q[D];
        alignas(16) uint16_t k[D];
        alignas(16) uint16_t v[D];
        alignas(16) float gate[D];
        alignas(16) uint8_t bits[D];
        alignas(16) float w[D];
    };
    Stage stage[2];
    alignas(16) float4 rc0[D];      // by key row i: alpha, alpha, alpha k, alpha k  (alpha = g r 2^(8-b))
    alignas(16) float4 rc1[D];      // by key row i: alpha q, alpha q, k, k
    alignas(16) float4 rq[D];       // by slot: e, e, G, G  (e = 1/(r~ 2^(8-b)), G = (w r~ 2^(8-b))^2)
    alignas(16) float riq[D];       // by slot: 1/q_b
    alignas(16) uint32_t meta[D];   // by slot: row | width << 8 | byte offset << 16
    alignas(16) float colc[D];      // c_j (old column scale)
    alignas(16) float colb[D];      // per-phase column broadcast
    alignas(16) float col0[D];      // c0_j
    alignas(16) float colm[D];      // max_i |xi_ij| / q_b
    alignas(16) float red[M::kWarps][2][D];
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
    alignas(8) uint64_t full[2];
    float qk;
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: a tile copy takes microseconds

template <int D>
__device__ __forceinline__ void issue_tile(const DecodeArgs& a, DecodeSmem<D>& sm, int n, int s) {
    const int tile = blockIdx.x + n * gridDim.x;
    if (tile >= a.num_tiles) return;
    const int b = tile / a.H, h = tile % a.H;
    const int64_t hoff = a.head_off[h];
    const int64_t hend = (h + 1 < a.H) ? a.head_off[h + 1] : a.bytes_per_seq;
    const uint32_t pbytes = static_cast<uint32_t>(hend - hoff);
    auto& st = sm.stage[s];
    const uint32_t total = pbytes + 5u * 2u * D + D + 4u * D + (a.gate_per_channel ? 4u * D : 0u);
    mbar_arrive_expect_tx(&sm.full[s], total);
    bulk_load(st.codes, a.packed_in + b * a.bytes_per_seq + hoff, pbytes, &sm.full[s]);
    bulk_load(st.r, a.r_in + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.c, a.c_in + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.q, a.q + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.k, a.k + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.v, a.v + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.bits, a.bits + static_cast<int64_t>(h) * D, D, &sm.full[s]);
    bulk_load(st.w, a.w + static_cast<int64_t>(h) * D, 4 * D, &sm.full[s]);
    if (a.gate_per_channel) bulk_load(st.gate, a.gate + static_cast<int64_t>(tile) * D, 4 * D, &sm.full[s]);
}

// Sort the rows of a tile by bit width (stable) and record, per slot, the row, its width and
// the byte offset of the row in the packed tile. One warp.
template <int D>
__device__ __forceinline__ void sort_rows_warp(const uint8_t* bits, uint32_t* meta, int lane) {
    constexpr int RL = D / 32;
    int bw[RL], loc[RL], rank[RL], sum = 0;
    int cnt[4] = {0, 0, 0, 0};
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        bw[r] = bits[lane * RL + r];
        loc[r] = sum;
        sum += bw[r] * (D / 8);
        const int cls = (bw[r] >> 1) - 1;
        rank[r] = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (c == cls) rank[r] = cnt[c];
            cnt[c] += (c == cls);
        }
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    int excl_c[4], base_c[4], base = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
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
        const int cls = (bw[r] >> 1) - 1;
        int slot = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c == cls) slot = base_c[c] + excl_c[c] + rank[r];
        const int off = incl - sum + loc[r];
        meta[slot] = static_cast<uint32_t>(lane * RL + r) | (static_cast<uint32_t>(bw[r]) << 8) |
                     (static_cast<uint32_t>(off) << 16);
    }
}

// ---- phase 1: unpack the thread's rows and accumulate the k^T and q^T products -------------
template <int D, int BW>
__device__ __forceinline__ void phase1_row(const DecodeSmem<D>& sm, const uint8_t* codes, uint32_t mt, int cl,
                                           float2& z01, float2& z23, float2 pacc[2], float2 oacc[2]) {
    const int i = mt & 0xFF;
    unpack4<D, BW>(codes + (mt >> 16), cl, z01, z23);
    const float4 c0 = sm.rc0[i], c1 = sm.rc1[i];
    const float2 kap = make_float2(c0.z, c0.w), lam = make_float2(c1.x, c1.y);
    pacc[0] = fma2(kap, z01, pacc[0]);
    pacc[1] = fma2(kap, z23, pacc[1]);
    oacc[0] = fma2(lam, z01, oacc[0]);
    oacc[1] = fma2(lam, z23, oacc[1]);
}

template <int D, int BW>
__device__ __forceinline__ void phase1_uniform(const DecodeSmem<D>& sm, const uint8_t* codes, int warp, int lane,
                                               float2 Z[][2], float2 pacc[2], float2 oacc[2]) {
    using M = Map<D>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r)
        phase1_row<D, BW>(sm, codes, sm.meta[M::row(warp, lane, r)], cl, Z[r][0], Z[r][1], pacc, oacc);
}

template <int D>
__device__ __forceinline__ void phase1_mixed(const DecodeSmem<D>& sm, const uint8_t* codes, int warp, int lane,
                                             float2 Z[][2], float2 pacc[2], float2 oacc[2]) {
    using M = Map<D>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const uint32_t mt = sm.meta[M::row(warp, lane, r)];
        switch ((mt >> 8) & 0xFF) {
            case 8: phase1_row<D, 8>(sm, codes, mt, cl, Z[r][0], Z[r][1], pacc, oacc); break;
            case 6: phase1_row<D, 6>(sm, codes, mt, cl, Z[r][0], Z[r][1], pacc, oacc); break;
            case 4: phase1_row<D, 4>(sm, codes, mt, cl, Z[r][0], Z[r][1], pacc, oacc); break;
            default: phase1_row<D, 2>(sm, codes, mt, cl, Z[r][0], Z[r][1], pacc, oacc); break;
        }
    }
}

// ---- phase 6: final codes, packed and stored ------------------------------------------------
template <int D, int BW, bool CLAMP>
__device__ __forceinline__ void phase6_row(uint8_t* out, uint32_t mt, int cl, float2 x01, float2 x23, float2 f01,
                                           float2 f23) {
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);
    const float2 a = fma2(x01, f01, M2), b = fma2(x23, f23, M2);
    pack4<D, BW, CLAMP>(out + (mt >> 16), cl, __float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x),
                        __float_as_uint(b.y));
}

template <int D, int BW, bool CLAMP>
__device__ __forceinline__ void phase6_uniform(const DecodeSmem<D>& sm, uint8_t* out, int warp, int lane,
                                               const float2 Z[][2], float2 f01, float2 f23) {
    using M = Map<D>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r)
        phase6_row<D, BW, CLAMP>(out, sm.meta[M::row(warp, lane, r)], cl, Z[r][0], Z[r][1], f01, f23);
}

template <int D, bool CLAMP>
__device__ __forceinline__ void phase6_mixed(const DecodeSmem<D>& sm, uint8_t* out, int warp, int lane,
                                             const float2 Z[][2], float2 f01, float2 f23) {
    using M = Map<D>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const uint32_t mt = sm.meta[M::row(warp, lane, r)];
        switch ((mt >> 8) & 0xFF) {
            case 8: phase6_row<D, 8, CLAMP>(out, mt, cl, Z[r][0], Z[r][1], f01, f23); break;
            case 6: phase6_row<D, 6, CLAMP>(out, mt, cl, Z[r][0], Z[r][1], f01, f23); break;
            case 4: phase6_row<D, 4, CLAMP>(out, mt, cl, Z[r][0], Z[r][1], f01, f23); break;
            default: phase6_row<D, 2, CLAMP>(out, mt, cl, Z[r][0], Z[r][1], f01, f23); break;
        }
    }
}

template <int D, bool CLAMP>
__device__ __forceinline__ void phase6(const DecodeSmem<D>& sm, uint8_t* out, int warp, int lane, int ww,
                                       const float2 Z[][2], float2 f01, float2 f23) {
    switch (ww) {
        case 8: phase6_uniform<D, 8, CLAMP>(sm, out, warp, lane, Z, f01, f23); break;
        case 6: phase6_uniform<D, 6, CLAMP>(sm, out, warp, lane, Z, f01, f23); break;
        case 4: phase6_uniform<D, 4, CLAMP>(sm, out, warp, lane, Z, f01, f23); break;
        case 2: phase6_uniform<D, 2, CLAMP>(sm, out, warp, lane, Z, f01, f23); break;
        default: phase6_mixed<D, CLAMP>(sm, out, warp, lane, Z, f01, f23); break;
    }
}

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads, Map<D>::kMinBlocks)
decode_kernel(const DecodeArgs a) {
    using M = Map<D>;
    constexpr int RPT = M::RPT;
    constexpr int LPR = M::LPR;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem<D>& sm = *reinterpret_cast<DecodeSmem<D>*>(smem_raw);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);

    if (tid == 0) {
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
        issue_tile<D>(a, sm, 0, 0);
    }
    __syncthreads();

    for (int n = 0;; ++n) {
        const int tile = blockIdx.x + n * gridDim.x;
        if (tile >= a.num_tiles) break;
        const int s = n & 1;
        const bool ok = mbar_wait_bounded(&sm.full[s], (n >> 1) & 1, kWaitLimitNs, &g_stepq_flags);
        if (__syncthreads_or(!ok)) {
            // A tile copy never arrived: give up (the host reads the error word), after one
            // more bounded wait for that copy, the only one in flight.
            if (tid == 0) mbar_wait_bounded(&sm.full[s], (n >> 1) & 1, kWaitLimitNs, &g_stepq_flags);
            return;
        }
        // Every thread is past the previous tile: its buffers may be refilled.
        if (tid == 0) issue_tile<D>(a, sm, n + 1, s ^ 1);

        auto& st = sm.stage[s];
        const int h = tile % a.H;
        const int64_t tile_base = static_cast<int64_t>(tile / a.H) * a.bytes_per_seq + a.head_off[h];

        // ---- prologue: per-row constants, width-sorted slots, q.k -----------------------
        if (tid < D) {
            const int i = tid;
            const int bw = st.bits[i];
            const float g = a.gate_per_channel ? st.gate[i] : __ldg(a.gate + tile);
            const float alpha = g * half_bits_to_float(st.r[i]) * znorm_of(bw);
            const float kk = bf16_bits_to_float(st.k[i]);
            const float qq = bf16_bits_to_float(st.q[i]);
            sm.rc0[i] = make_float4(alpha, alpha, alpha * kk, alpha * kk);
            sm.rc1[i] = make_float4(alpha * qq, alpha * qq, kk, kk);
        } else if (warp == D / 32) {
            sort_rows_warp<D>(st.bits, sm.meta, lane);
        } else if (warp == D / 32 + 1) {
            constexpr int RL = D / 32;
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < RL; ++r)
                acc = fmaf(bf16_bits_to_float(st.q[lane * RL + r]), bf16_bits_to_float(st.k[lane * RL + r]), acc);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) sm.qk = acc;
        }
        __syncthreads();

        // The warp's 16 slots share one width unless the warp straddles a width boundary.
        int ww;
        {
            const int w0 = (sm.meta[warp * M::kRowsPerWarp] >> 8) & 0xFF;
            const int w1 = (sm.meta[warp * M::kRowsPerWarp + M::kRowsPerWarp - 1] >> 8) & 0xFF;
            ww = (w0 == w1) ? w0 : 0;
        }

        // ---- phase 1: unpack, k^T D S and q^T D S (column scale factored out) ----------
        float2 Z[RPT][2];
        float2 pacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 oacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        switch (ww) {
            case 8: phase1_uniform<D, 8>(sm, st.codes, warp, lane, Z, pacc, oacc); break;
            case 6: phase1_uniform<D, 6>(sm, st.codes, warp, lane, Z, pacc, oacc); break;
            case 4: phase1_uniform<D, 4>(sm, st.codes, warp, lane, Z, pacc, oacc); break;
            case 2: phase1_uniform<D, 2>(sm, st.codes, warp, lane, Z, pacc, oacc); break;
            default: phase1_mixed<D>(sm, st.codes, warp, lane, Z, pacc, oacc); break;
        }
#pragma unroll
        for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                pacc[q2].x += __shfl_xor_sync(0xffffffffu, pacc[q2].x, m);
                pacc[q2].y += __shfl_xor_sync(0xffffffffu, pacc[q2].y, m);
                oacc[q2].x += __shfl_xor_sync(0xffffffffu, oacc[q2].x, m);
                oacc[q2].y += __shfl_xor_sync(0xffffffffu, oacc[q2].y, m);
            }
        if (lane < LPR) {
            *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(pacc[0].x, pacc[0].y, pacc[1].x, pacc[1].y);
            *reinterpret_cast<float4*>(&sm.red[warp][1][4 * cl]) = make_float4(oacc[0].x, oacc[0].y, oacc[1].x, oacc[1].y);
        }
        __syncthreads();

        // ---- phase 2: u = beta (v - k^T D S), o = q^T X ---------------------------------
        if (tid < D) {
            const int j = tid;
            float ps = 0.f, os = 0.f;
#pragma unroll
            for (int w = 0; w < M::kWarps; ++w) {
                ps += sm.red[w][0][j];
                os += sm.red[w][1][j];
            }
            const float cj = half_bits_to_float(st.c[j]);
            const float beta = __ldg(a.beta + tile);
            const float u = beta * (bf16_bits_to_float(st.v[j]) - cj * ps);
            a.o[static_cast<int64_t>(tile) * D + j] = fmaf(cj, os, sm.qk * u);
            sm.colc[j] = cj;
            sm.colb[j] = u / cj;
        }
        __syncthreads();

        // ---- phase 3: X = D S + k u^T (divided by c_j), row |.| sums --------------------
        const float4 c4 = *reinterpret_cast<const float4*>(&sm.colc[4 * cl]);
        {
            const float4 u4 = *reinterpret_cast<const float4*>(&sm.colb[4 * cl]);
            const float2 ut01 = make_float2(u4.x, u4.y), ut23 = make_float2(u4.z, u4.w);
            float part[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int i = sm.meta[M::row(warp, lane, r)] & 0xFF;
                const float4 c0 = sm.rc0[i], c1 = sm.rc1[i];
                const float2 al = make_float2(c0.x, c0.y), kk = make_float2(c1.z, c1.w);
                Z[r][0] = fma2(al, Z[r][0], mul2(kk, ut01));
                Z[r][1] = fma2(al, Z[r][1], mul2(kk, ut23));
                float acc = fabsf(Z[r][0].x) * c4.x;
                acc = fmaf(fabsf(Z[r][0].y), c4.y, acc);
                acc = fmaf(fabsf(Z[r][1].x), c4.z, acc);
                part[r] = fmaf(fabsf(Z[r][1].y), c4.w, acc);
            }
            int slot;
            bool owner;
            const float rsum = row_reduce<D, float>(sm.rowbuf[warp], lane, part, slot, OpAdd());
            const int sl = reduced_row<D>(warp, lane, slot, owner);   // a slot index here
            if (owner) {
                const uint32_t mt = sm.meta[sl];
                const int i = mt & 0xFF, bw = (mt >> 8) & 0xFF;
                const float wi = st.w[i];
                const __half rh = scale_to_half(fmaxf(rsum * (1.0f / D), kHalfMinNormal) / wi);
                a.r_out[static_cast<int64_t>(tile) * D + i] = __half_as_ushort(rh);
                const float rs = __half2float(rh) * znorm_of(bw);
                const float e = __frcp_rn(rs);
                const float g = wi * rs;
                sm.rq[sl] = make_float4(e, e, g * g, g * g);
                sm.riq[sl] = __frcp_rn(static_cast<float>(qmax_of(bw)));
            }
            __syncwarp();
        }

        // ---- phase 4: xi = X / (c_j r~_i 2^(8-b_i)); column no-clip scale c0 -----------
        {
            float cmax[4] = {0.f, 0.f, 0.f, 0.f};
            if (ww != 0) {
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float4 q4 = sm.rq[M::row(warp, lane, r)];
                    const float2 e2 = make_float2(q4.x, q4.y);
                    Z[r][0] = mul2(Z[r][0], e2);
                    Z[r][1] = mul2(Z[r][1], e2);
                    cmax[0] = fmaxf(cmax[0], fabsf(Z[r][0].x));
                    cmax[1] = fmaxf(cmax[1], fabsf(Z[r][0].y));
                    cmax[2] = fmaxf(cmax[2], fabsf(Z[r][1].x));
                    cmax[3] = fmaxf(cmax[3], fabsf(Z[r][1].y));
                }
                const float iq = sm.riq[warp * M::kRowsPerWarp];
#pragma unroll
                for (int kx = 0; kx < 4; ++kx) cmax[kx] *= iq;
            } else {
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int sl = M::row(warp, lane, r);
                    const float4 q4 = sm.rq[sl];
                    const float2 e2 = make_float2(q4.x, q4.y);
                    const float iq = sm.riq[sl];
                    Z[r][0] = mul2(Z[r][0], e2);
                    Z[r][1] = mul2(Z[r][1], e2);
                    cmax[0] = fmaxf(cmax[0], fabsf(Z[r][0].x) * iq);
                    cmax[1] = fmaxf(cmax[1], fabsf(Z[r][0].y) * iq);
                    cmax[2] = fmaxf(cmax[2], fabsf(Z[r][1].x) * iq);
                    cmax[3] = fmaxf(cmax[3], fabsf(Z[r][1].y) * iq);
                }
            }
            combine_subrows<D, float>(cmax, OpMax());
            if (lane < LPR)
                *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(cmax[0], cmax[1], cmax[2], cmax[3]);
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
            sm.colm[j] = cm;
            sm.colb[j] = cj / c0;
        }
        __syncthreads();

        // ---- phase 5: codes at (r~, c0); weighted least-squares column update ----------
        {
            const float4 f4 = *reinterpret_cast<const float4*>(&sm.colb[4 * cl]);
            const float2 f01 = make_float2(f4.x, f4.y), f23 = make_float2(f4.z, f4.w);
            const float2 mM2 = make_float2(-kRoundMagic, -kRoundMagic);
            float2 num[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float2 den[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float4 q4 = sm.rq[M::row(warp, lane, r)];
                const float2 G2 = make_float2(q4.z, q4.w);
                const float2 z01 = add2(fma2(Z[r][0], f01, M2), mM2);
                const float2 z23 = add2(fma2(Z[r][1], f23, M2), mM2);
                const float2 g01 = mul2(G2, z01), g23 = mul2(G2, z23);
                num[0] = fma2(g01, Z[r][0], num[0]);
                num[1] = fma2(g23, Z[r][1], num[1]);
                den[0] = fma2(g01, z01, den[0]);
                den[1] = fma2(g23, z23, den[1]);
            }
#pragma unroll
            for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    num[q2].x += __shfl_xor_sync(0xffffffffu, num[q2].x, m);
                    num[q2].y += __shfl_xor_sync(0xffffffffu, num[q2].y, m);
                    den[q2].x += __shfl_xor_sync(0xffffffffu, den[q2].x, m);
                    den[q2].y += __shfl_xor_sync(0xffffffffu, den[q2].y, m);
                }
            if (lane < LPR) {
                *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(num[0].x, num[0].y, num[1].x, num[1].y);
                *reinterpret_cast<float4*>(&sm.red[warp][1][4 * cl]) = make_float4(den[0].x, den[0].y, den[1].x, den[1].y);
            }
        }
        __syncthreads();
        bool clip = false;
        if (tid < D) {
            const int j = tid;
            float ns = 0.f, ds = 0.f;
#pragma unroll
            for (int w = 0; w < M::kWarps; ++w) {
                ns += sm.red[w][0][j];
                ds += sm.red[w][1][j];
            }
            const float cj = sm.colc[j];
            const float c1 = ds > 0.f ? (cj * ns) / ds : sm.col0[j];
            const __half ch = scale_to_half(c1);
            a.c_out[static_cast<int64_t>(tile) * D + j] = __half_as_ushort(ch);
            const float fq = cj / __half2float(ch);
            sm.colb[j] = fq;
            // |t_ij| <= q_b max_i(|xi_ij|/q_b) fq_j: past this margin a code may round beyond q_b.
            clip = sm.colm[j] * fq > 1.0f + 0.4f / 127.0f;
        }
        const bool any_clip = __syncthreads_or(clip);

        // ---- phase 6: final codes at (r~, c~), packed and stored -----------------------
        {
            const float4 f4 = *reinterpret_cast<const float4*>(&sm.colb[4 * cl]);
            const float2 f01 = make_float2(f4.x, f4.y), f23 = make_float2(f4.z, f4.w);
            uint8_t* out = a.packed_out + tile_base;
            if (any_clip) phase6<D, true>(sm, out, warp, lane, ww, Z, f01, f23);
            else phase6<D, false>(sm, out, warp, lane, ww, Z, f01, f23);
        }
    }
}

template <int D>
static int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    static int ctas_per_sm = -1, num_sms = 0;
    const size_t smem = sizeof(DecodeSmem<D>);
    if (ctas_per_sm < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        int occ = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<D>, Map<D>::kThreads, smem);
        ctas_per_sm = occ > 0 ? occ : 1;
    }
    if (a.num_tiles == 0) return STEPQ_OK;
    int grid = num_sms * ctas_per_sm;
    if (grid > a.num_tiles) grid = a.num_tiles;
    decode_kernel<D><<<grid, Map<D>::kThreads, smem, stream>>>(a);
    return check_launch("stepq_decode_step");
}

}  // namespace stepq

using namespace stepq;

extern "C" int stepq_decode_step(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const float* beta, const float* gate, const uint8_t* bits, const float* w,
                                 const int64_t* head_off, int64_t bytes_per_seq, const uint8_t* packed_in,
                                 const uint16_t* r_in, const uint16_t* c_in, uint8_t* packed_out,
                                 uint16_t* r_out, uint16_t* c_out, float* o, void* stream) {
    clear_error();
    int rc = check_dims(dims, "stepq_decode_step");
    if (rc) return rc;
    if (dims.B == 0) return STEPQ_OK;
    rc = check_ptrs("stepq_decode_step", {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate},
                                          {"bits", bits}, {"w", w}, {"head_off", head_off},
                                          {"packed_in", packed_in}, {"r_in", r_in}, {"c_in", c_in},
                                          {"packed_out", packed_out}, {"r_out", r_out}, {"c_out", c_out},
                                          {"o", o}});
    if (rc) return rc;
    if (bytes_per_seq <= 0 || (bytes_per_seq & 15))
        return set_error(STEPQ_EINVAL, "stepq_decode_step: bytes_per_seq=%lld", (long long)bytes_per_seq);
    const long long tiles = static_cast<long long>(dims.B) * dims.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "stepq_decode_step: too many tiles");
    DecodeArgs a{dims.B, dims.H, dims.gate_per_channel, static_cast<int>(tiles), q, k, v, beta, gate, bits, w,
                 head_off, bytes_per_seq, packed_in, r_in, c_in, packed_out, r_out, c_out, o};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128 ? launch_decode<128>(a, st) : launch_decode<64>(a, st);
}

extern "C" int stepq_read_device_flags(uint32_t* flags_host) {
    clear_error();
    if (!flags_host) return set_error(STEPQ_EINVAL, "stepq_read_device_flags: null output");
    uint32_t zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(flags_host, g_stepq_flags, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_stepq_flags, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "stepq_read_device_flags: %s", cudaGetErrorString(e));
    return STEPQ_OK;
}
