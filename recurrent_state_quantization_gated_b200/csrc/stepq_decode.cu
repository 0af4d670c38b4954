// stepq_decode.cu -- the fused quantized decode step (STEPQuant, Table C2) for sm_100a.
//
// One persistent CTA per SM slot walks over (sequence, head) tiles. The frozen bit map is
// turned once per launch into per-head tables (rows sorted by width, byte offsets, row-impact
// factors) kept in shared memory. For each tile the bulk-copy (TMA) engine stages the packed
// codes, the old scales, q/k/v and the gate into shared memory, double buffered so that the
// next tile's copy runs while this one is computed. The tile then lives in registers (a thread
// owns 8 columns of D/16 rows) through every phase:
//   1 unpack + dequantise (the column scale is factored out: Xi_ij = X_ij / c_j), and the two
//     column dot products k^T D S and q^T D S of the Delta rule;
//   2 u = beta (v - k^T D S), o = q^T X = q^T D S + (q.k) u          (§2.1, Table C2 step 3);
//   3 X = D S + k u^T and the row factors m_i = mean_j |X_ij|        (§4.3 "Row factors");
//   4 the no-clip column initialisation c0_j                         (fit start);
//   5 codes at (r, c0) and the weighted least-squares column update   (App. C.1);
//   6 final codes at (r, c), packed and stored straight to HBM.
// Rows are visited sorted by bit width, so almost every warp runs a width-specialised unpack
// and pack; floating-point work runs on packed f32x2 instructions. Column reductions cross
// warps through shared memory, row reductions stay inside a warp. The state is read from HBM
// once and written once; no tensor cores (a rank-1 update per token is not a dense
// contraction).
#include <cuda_runtime.h>

#include <mutex>

#include "stepq_device.cuh"
#include "stepq_tile.cuh"
#include "stepq_internal.h"

namespace stepq {

// Device error word: bit 0 = a bounded wait for a tile copy gave up; bit 1 = an FP16 pivot row
// in a launch declared without pivots; bit 2 = a head range that cannot hold its tile.
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
    float* x_out;   // split form only: the updated state X [B][H][dk][dv] before requantisation
    int chunk;      // tokens per launch (1: one decode step; > 1: a prefill chunk, inputs and o
                    // with a leading token axis)
};

constexpr int kStages = 3;   // tile copies in flight: the current tile and the next two

// Sorted-row tables of heads kept in shared memory: a direct-mapped cache (head h lives in
// entry h % kHeads), filled when a tile of a head not held is decoded. With at most kHeads
// heads every table is built once per CTA and launch.
template <int D>
struct HeadCache {
    static constexpr int kHeads = (D == 128) ? 32 : 64;
};

template <int D>
struct DecodeSmem {
    using M = DMap<D>;
    static constexpr int CH = HeadCache<D>::kHeads;
    struct Stage {
        alignas(16) uint8_t codes[D * D];   // room for an all-8-bit tile
        alignas(16) uint16_t r[D];
        alignas(16) uint16_t c[D];
        alignas(16) uint16_t q[D];
        alignas(16) uint16_t k[D];
        alignas(16) uint16_t v[D];
        alignas(16) float gate[D];
        alignas(16) float w[D];
        float beta;                          // scalars of this tile, prefetched with it
        float gate1;
    };
    Stage stage[kStages];
    // Per head (cached): per slot (rows sorted by width, stable) the row's metadata
    // row | width << 8 | byte offset << 16.
    alignas(16) uint32_t hmeta[CH][D];
    alignas(16) uint16_t hslot[CH][D];   // by key row: slot | width << 8
    int htag[CH];                   // head held by each cache entry (-1: none)
    int hok[CH];                    // the head's byte range holds its tile under the bit map
    long long hoff[CH];             // head_off of the head
    // Per slot of the tile being decoded.
    alignas(16) float4 kq[D];       // alpha k, alpha k, alpha q, alpha q   (alpha = g r 2^(8-b))
    alignas(16) float4 ak[2][D];    // k/alpha, k/alpha, alpha, alpha (two tokens of a chunk)
    alignas(16) float4 rq[D];       // alpha e, alpha e, G, G  (e = 1/(r~ 2^(8-b)), G = (w r~ 2^(8-b))^2)
    alignas(16) float2 wsl[D];      // w, 1/w
    alignas(16) float riq[D];       // 1/q_b
    // Per column.
    alignas(16) float colc[D];      // c_j (old column scale)
    alignas(16) float icol[D];      // 1/c_j (FP16 pivot rows enter the tile as x / c_j)
    alignas(16) float colb[D];      // per-phase column broadcast
    alignas(16) float col0[D];      // c0_j
    alignas(16) float red[M::kWarps][2][D];
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
    alignas(8) uint64_t full[kStages];
    float qk;
    float qkp[2][D / 32];           // q.k of a chunk's token, one partial per 32 key rows
    int rn[2][D / 32];              // a chunk's token renormalises some key row's gate product
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: a tile copy takes microseconds

// Queue the bulk copies of `tile` into stage s (one thread). The tile's two scalars are
// returned in registers for the caller to store later, so their load latency stays hidden.
template <int D>
__device__ __forceinline__ bool issue_tile(const DecodeArgs& a, DecodeSmem<D>& sm, int tile, int s, float& beta,
                                           float& gate1) {
    if (tile >= a.num_tiles) return false;
    const int b = tile / a.H, h = tile % a.H;
    int64_t hoff, hend;
    // The stage holds the integer rows (at most D*D bytes); FP16 pivot rows, stored after them,
    // are read from global memory where they are used. A head range that cannot hold a tile
    // copies no codes (the tile is skipped where it is computed).
    const bool range_ok = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, -1, 2 * D * D, &g_stepq_flags, &hoff, &hend);
    const uint32_t pbytes = range_ok ? static_cast<uint32_t>(min(hend - hoff, static_cast<int64_t>(D) * D)) : 0u;
    auto& st = sm.stage[s];
    const uint32_t total = pbytes + 5u * 2u * D + 4u * D + (a.gate_per_channel ? 4u * D : 0u);
    mbar_arrive_expect_tx(&sm.full[s], total);
    if (pbytes) bulk_load(st.codes, a.packed_in + b * a.bytes_per_seq + hoff, pbytes, &sm.full[s]);
    bulk_load(st.r, a.r_in + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.c, a.c_in + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.q, a.q + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.k, a.k + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.v, a.v + static_cast<int64_t>(tile) * D, 2 * D, &sm.full[s]);
    bulk_load(st.w, a.w + static_cast<int64_t>(h) * D, 4 * D, &sm.full[s]);
    if (a.gate_per_channel) bulk_load(st.gate, a.gate + static_cast<int64_t>(tile) * D, 4 * D, &sm.full[s]);
    beta = __ldg(a.beta + tile);
    gate1 = a.gate_per_channel ? 0.f : __ldg(a.gate + tile);
    return true;
}

// The n-th tile of this CTA (tiles are dealt round-robin over the persistent CTAs).
__device__ __forceinline__ int cta_tile(int n) { return blockIdx.x + n * gridDim.x; }

// ---- phase 1: unpack the thread's rows and accumulate the k^T and q^T products -------------
template <int D, int BW>
__device__ __forceinline__ void phase1_row(const DecodeSmem<D>& sm, const uint8_t* codes, int s, uint32_t mt,
                                           int cl, float2 z[4], float2 pacc[4], float2 oacc[4]) {
    unpack8<D, BW>(codes + (mt >> 16), cl, z);
    const float4 c = sm.kq[s];
    const float2 kap = make_float2(c.x, c.y), lam = make_float2(c.z, c.w);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        pacc[p] = fma2(kap, z[p], pacc[p]);
        oacc[p] = fma2(lam, z[p], oacc[p]);
    }
}

// An FP16 pivot row: eight values, divided by their column scales so that the row joins the
// tile's factored form X = alpha_i c_j Y_ij with alpha_i = g_i. Pivot rows follow the integer
// rows of a tile: those inside the staged first d*d bytes are read from shared memory, the
// rest from global memory (a generic load serves both).
template <int D>
__device__ __forceinline__ void load_pivot8(const uint8_t* row, int cl, const float* icol, float2 z[4]) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + 16 * cl);
    const float4 i0 = *reinterpret_cast<const float4*>(icol + 8 * cl);
    const float4 i1 = *reinterpret_cast<const float4*>(icol + 8 * cl + 4);
    z[0] = mul2(__half22float2(*reinterpret_cast<const __half2*>(&u.x)), make_float2(i0.x, i0.y));
    z[1] = mul2(__half22float2(*reinterpret_cast<const __half2*>(&u.y)), make_float2(i0.z, i0.w));
    z[2] = mul2(__half22float2(*reinterpret_cast<const __half2*>(&u.z)), make_float2(i1.x, i1.y));
    z[3] = mul2(__half22float2(*reinterpret_cast<const __half2*>(&u.w)), make_float2(i1.z, i1.w));
}

template <int D>
__device__ __forceinline__ void phase1_pivot_row(const DecodeSmem<D>& sm, const uint8_t* codes, const uint8_t* gin,
                                                 int s, uint32_t mt, int cl, float2 z[4], float2 pacc[4],
                                                 float2 oacc[4]) {
    const uint32_t off = mt >> 16;
    load_pivot8<D>((off + 2 * D <= D * D ? codes : gin) + off, cl, sm.icol, z);
    const float4 c = sm.kq[s];
    const float2 kap = make_float2(c.x, c.y), lam = make_float2(c.z, c.w);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        pacc[p] = fma2(kap, z[p], pacc[p]);
        oacc[p] = fma2(lam, z[p], oacc[p]);
    }
}

template <int D>
__device__ __forceinline__ void phase1_pivots(const DecodeSmem<D>& sm, const uint32_t* meta, const uint8_t* codes,
                                              const uint8_t* gin, int warp, int lane, float2 Z[][4], float2 pacc[4],
                                              float2 oacc[4]) {
    using M = DMap<D>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int s = M::row(warp, lane, r);
        phase1_pivot_row<D>(sm, codes, gin, s, meta[s], cl, Z[r], pacc, oacc);
    }
}

// Width-uniform warp: every row's metadata and code words are loaded first, so the shared
// memory latencies overlap, then the rows are unpacked and accumulated.
template <int D, int BW>
__device__ __forceinline__ void phase1_uniform(const DecodeSmem<D>& sm, const uint32_t* meta, const uint8_t* codes,
                                               int warp, int lane, float2 Z[][4], float2 pacc[4], float2 oacc[4]) {
    using M = DMap<D>;
    const int cl = M::col_lane(lane);
    uint32_t mt[M::RPT];
    uint2 raw[M::RPT];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) mt[r] = meta[M::row(warp, lane, r)];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) raw[r] = load8<D, BW>(codes + (mt[r] >> 16), cl);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        unpack8r<BW>(raw[r], Z[r]);
        const float4 c = sm.kq[M::row(warp, lane, r)];
        const float2 kap = make_float2(c.x, c.y), lam = make_float2(c.z, c.w);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            pacc[p] = fma2(kap, Z[r][p], pacc[p]);
            oacc[p] = fma2(lam, Z[r][p], oacc[p]);
        }
    }
}

template <int D, bool kPiv, int kW = 0>
__device__ __forceinline__ void phase1_mixed(const DecodeSmem<D>& sm, const uint32_t* meta, const uint8_t* codes,
                                             const uint8_t* gin, int warp, int lane, float2 Z[][4], float2 pacc[4],
                                             float2 oacc[4]) {
    using M = DMap<D>;
    using WS = WidthSet<kW>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int s = M::row(warp, lane, r);
        const uint32_t mt = meta[s];
        const int bw = (mt >> 8) & 0xFF;
        if constexpr (WS::tested(8)) if (bw == 8) { phase1_row<D, 8>(sm, codes, s, mt, cl, Z[r], pacc, oacc); continue; }
        if constexpr (WS::tested(6)) if (bw == 6) { phase1_row<D, 6>(sm, codes, s, mt, cl, Z[r], pacc, oacc); continue; }
        if constexpr (WS::tested(4)) if (bw == 4) { phase1_row<D, 4>(sm, codes, s, mt, cl, Z[r], pacc, oacc); continue; }
        if constexpr (WS::tested(2)) if (bw == 2) { phase1_row<D, 2>(sm, codes, s, mt, cl, Z[r], pacc, oacc); continue; }
        if constexpr (kPiv) if (bw == 16) { phase1_pivot_row<D>(sm, codes, gin, s, mt, cl, Z[r], pacc, oacc); continue; }
        phase1_row<D, WS::fallback>(sm, codes, s, mt, cl, Z[r], pacc, oacc);
    }
}

template <int D, bool kPiv, int kW = 0>
__device__ __forceinline__ void phase1(const DecodeSmem<D>& sm, const uint32_t* meta, const uint8_t* codes,
                                       const uint8_t* gin, int warp, int lane, int ww, float2 Z[][4],
                                       float2 pacc[4], float2 oacc[4]) {
    switch (ww) {
        case 8: phase1_uniform<D, 8>(sm, meta, codes, warp, lane, Z, pacc, oacc); break;
        case 6: phase1_uniform<D, 6>(sm, meta, codes, warp, lane, Z, pacc, oacc); break;
        case 4: phase1_uniform<D, 4>(sm, meta, codes, warp, lane, Z, pacc, oacc); break;
        case 2: phase1_uniform<D, 2>(sm, meta, codes, warp, lane, Z, pacc, oacc); break;
        default:
            if constexpr (kPiv) {
                if (ww == 16) {
                    phase1_pivots<D>(sm, meta, codes, gin, warp, lane, Z, pacc, oacc);
                    break;
                }
            }
            phase1_mixed<D, kPiv, kW>(sm, meta, codes, gin, warp, lane, Z, pacc, oacc);
            break;
    }
}

// A prefill token's inputs as one thread needs them: key row i's k, q and gate (the thread
// writing row i's constants) or column j's v and the token's beta (the thread finalising
// column j). Inputs carry a leading token axis of T tiles each.
template <int D>
struct TokenRow {
    float k = 0.f, q = 0.f, g = 0.f;
    __device__ __forceinline__ void load(const DecodeArgs& a, int64_t T, int tile, int i, int t) {
        const int64_t tt = t * T + tile, ti = tt * D + i;
        k = bf16_bits_to_float(__ldg(a.k + ti));
        q = bf16_bits_to_float(__ldg(a.q + ti));
        g = a.gate_per_channel ? __ldg(a.gate + ti) : __ldg(a.gate + tt);
    }
};
template <int D>
struct TokenCol {
    float v = 0.f, beta = 0.f;
    __device__ __forceinline__ void load(const DecodeArgs& a, int64_t T, int tile, int j, int t) {
        const int64_t tt = t * T + tile;
        v = bf16_bits_to_float(__ldg(a.v + tt * D + j));
        beta = __ldg(a.beta + tt);
    }
};

// Per-slot constants of prefill token t for key row i (alpha_t = g_t alpha_{t-1}), written by
// the D threads that are not finalising columns; their warps reduce q.k partials. A row whose
// gate product falls below 2^-32 is renormalised: its Y is scaled by that product and alpha
// restarts at 1 (ak.w holds the scale, 1 otherwise), so that no product over a chunk, however
// long or steep its gates, leaves fp32 range or is floored.
template <int D>
__device__ __forceinline__ void token_constants(DecodeSmem<D>& sm, int he, int i, int t, const TokenRow<D>& in) {
    const int sl = sm.hslot[he][i] & 0xFF;
    const float raw = in.g * sm.ak[(t - 1) & 1][sl].z;
    const bool renorm = raw < 0x1p-32f;
    const float alpha = renorm ? 1.0f : raw;
    sm.kq[sl] = make_float4(alpha * in.k, alpha * in.k, alpha * in.q, alpha * in.q);
    const float ka = in.k * rcp_approx(alpha);
    sm.ak[t & 1][sl] = make_float4(ka, ka, alpha, renorm ? raw : 1.0f);
    const bool any = __any_sync(0xffffffffu, renorm);
    float qk = in.q * in.k;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);
    if ((i & 31) == 0) {
        sm.qkp[t & 1][i >> 5] = qk;
        sm.rn[t & 1][i >> 5] = any;
    }
}

// The tile loop of the decode kernel. kPiv: the bit map may hold FP16 pivot rows (declared by
// the caller in stepq_dims.pivots); launches without them run the leaner instantiation. A
// width-16 row met in a launch declared without pivots raises bit 1 of the device error word.
template <int D, bool kSplit, bool kPiv, bool kChunk, bool kMixed, int kW>
__device__ __forceinline__ void run_tiles(const DecodeArgs& a, DecodeSmem<D>& sm) {
    using M = DMap<D>;
    constexpr int RPT = M::RPT;
    constexpr int CH = HeadCache<D>::kHeads;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);
    const bool issuer = (tid == M::kThreads - 1);
    // The tile's (sequence, head) and stage, stepped per tile instead of divided out.
    const int step_b = gridDim.x / a.H, step_h = gridDim.x % a.H;
    int seq = blockIdx.x / a.H, h = blockIdx.x % a.H;
    int s = 0;
    uint32_t parity = 0;
    for (int n = 0;; ++n) {
        if (n > 0) {
            seq += step_b;
            h += step_h;
            if (h >= a.H) { h -= a.H; ++seq; }
            if (++s == kStages) { s = 0; parity ^= 1u; }
        }
        const int tile = cta_tile(n);
        if (tile >= a.num_tiles) break;
        const auto& st = sm.stage[s];
        const int he = h % CH;
        const uint32_t* meta = sm.hmeta[he];
        if (sm.htag[he] != h) {                     // every warp sees the same tag: uniform branch
            __syncthreads();                        // nobody still reads the entry
            if (warp == 0) {
                const int tot = sort_head_rows<D, kPiv>(a.bits + static_cast<int64_t>(h) * D, sm.hmeta[he],
                                                        sm.hslot[he], lane, &g_stepq_flags);
                if (lane == 0) {
                    int64_t ho, hn;
                    sm.hok[he] = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, tot, 2 * D * D, &g_stepq_flags, &ho, &hn);
                    sm.hoff[he] = ho;
                    sm.htag[he] = h;
                }
            }
            __syncthreads();
        }
        const bool tile_ok = sm.hok[he];
        const int64_t tile_base = static_cast<int64_t>(seq) * a.bytes_per_seq + sm.hoff[he];
        const bool ok = mbar_wait_bounded(&sm.full[s], parity, kWaitLimitNs, &g_stepq_flags);

        // A prefill chunk's token 1: its inputs are loaded now, behind the unpack (rows by the
        // threads tid >= D, columns by the threads tid < D); later tokens one window ahead.
        TokenRow<D> rowA;
        TokenCol<D> colA;
        if constexpr (kChunk) {
            if (a.chunk > 1) {
                if (tid >= D) rowA.load(a, a.num_tiles, tile, tid - D, 1);
                else colA.load(a, a.num_tiles, tile, tid, 1);
            }
        }

        // ---- prologue: per-slot constants of this tile, q.k ------------------------------
        if (ok && tile_ok) {
            if (tid < D) {
                const int i = tid;
                const uint32_t sw = sm.hslot[he][i];
                const int sl = sw & 0xFF, bw = sw >> 8;
                const float g = a.gate_per_channel ? st.gate[i] : st.gate1;
                // alpha > 0 always (a zero gate leaves 2^-64: far below any term that counts);
                // an FP16 pivot row carries its values, so alpha is the gate alone.
                const float alpha = fmaxf(kPiv && bw == 16 ? g : g * half_bits_to_float(st.r[i]) * znorm_of(bw), 0x1p-64f);
                const float kk = bf16_bits_to_float(st.k[i]);
                const float qq = bf16_bits_to_float(st.q[i]);
                const float wi = st.w[i];
                const float ka = kk * rcp_approx(alpha);
                sm.kq[sl] = make_float4(alpha * kk, alpha * kk, alpha * qq, alpha * qq);
                sm.ak[0][sl] = make_float4(ka, ka, alpha, alpha);
                sm.wsl[sl] = make_float2(wi, rcp_approx(wi));
                if constexpr (kPiv) sm.icol[i] = rcp_approx(half_bits_to_float(st.c[i]));   // column i
            } else if (warp == D / 32) {
                constexpr int RL = D / 32;
                float acc = 0.f;
#pragma unroll
                for (int r = 0; r < RL; ++r)
                    acc = fmaf(bf16_bits_to_float(st.q[lane * RL + r]), bf16_bits_to_float(st.k[lane * RL + r]), acc);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (lane == 0) sm.qk = acc;
            }
        }
        if (__syncthreads_or(!ok)) {
            // A tile copy never arrived: give up (the host reads the error word), after one
            // more bounded wait for each copy still in flight.
            if (issuer)
                for (int i = 0; i + 1 < kStages; ++i)
                    if (cta_tile(n + i) < a.num_tiles)
                        mbar_wait_bounded(&sm.full[(n + i) % kStages], ((n + i) / kStages) & 1, kWaitLimitNs,
                                          &g_stepq_flags);
            return;
        }
        // Every thread is past the previous tile, so its stage may be refilled kStages-1 ahead;
        // the copies are queued below while half of the CTA finalises the first reductions.
        const int ahead = n + kStages - 1, sa = s == 0 ? kStages - 1 : s - 1;   // ahead % kStages
        bool issued = false;
        float next_beta = 0.f, next_gate = 0.f;
        if (!tile_ok) {   // uniform: nothing of this tile is read or written
            if (issuer && issue_tile<D>(a, sm, cta_tile(ahead), sa, next_beta, next_gate)) {
                sm.stage[sa].beta = next_beta;
                sm.stage[sa].gate1 = next_gate;
            }
            __syncthreads();
            continue;
        }

        // The warp's 16 slots share one width unless the warp straddles a width boundary.
        int ww;
        {
            const int w0 = (meta[warp * M::kRowsPerWarp] >> 8) & 0xFF;
            const int w1 = (meta[warp * M::kRowsPerWarp + M::kRowsPerWarp - 1] >> 8) & 0xFF;
            ww = (!kMixed && w0 == w1) ? w0 : 0;   // kMixed: one code path for every width
        }

        // ---- phase 1: unpack, k^T D S and q^T D S (column scale factored out) ----------
        float2 Z[RPT][4];
        {
            float2 pacc[4], oacc[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) pacc[p] = oacc[p] = make_float2(0.f, 0.f);
            phase1<D, kPiv, kW>(sm, meta, st.codes, a.packed_in + tile_base, warp, lane, ww, Z, pacc, oacc);
            store_col_partials<D>(sm.red[warp][0], lane, pacc);
            store_col_partials<D>(sm.red[warp][1], lane, oacc);
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
            const float u = st.beta * (bf16_bits_to_float(st.v[j]) - cj * ps);
            a.o[static_cast<int64_t>(tile) * D + j] = fmaf(cj, os, sm.qk * u);
            sm.colc[j] = cj;
            sm.colb[j] = u * rcp_approx(cj);
        } else {
            if (issuer) issued = issue_tile<D>(a, sm, cta_tile(ahead), sa, next_beta, next_gate);
            if constexpr (kChunk) {
                if (a.chunk > 1) {   // token 1's constants, while token 0 is finalised
                    token_constants<D>(sm, he, tid - D, 1, rowA);
                    if (a.chunk > 2) rowA.load(a, a.num_tiles, tile, tid - D, 2);
                }
            }
        }
        __syncthreads();

        // ---- prefill chunk: tokens 1 .. C-1 in full precision on the register-resident tile
        //      (no requantisation between them); the gate folds into alpha_i ---------------
        int kb = 0;   // the buffer of ak holding the last token's k/alpha and alpha
        if constexpr (kChunk) {
            const int64_t T = a.num_tiles;
            for (int t = 1; t < a.chunk; ++t) {
                bool rn = false;   // some row's gate product renormalised at token t (uniform)
#pragma unroll
                for (int w = 0; w < D / 32; ++w) rn |= sm.rn[t & 1][w] != 0;
                {   // token t-1's rank-1 update fused with token t's k^T X and q^T X (and, where
                    // token t renormalises a row's gate product, its scaling in between)
                    float2 ut[4], pacc[4], oacc[4];
                    load_cols8(sm.colb, cl, ut);
#pragma unroll
                    for (int p = 0; p < 4; ++p) pacc[p] = oacc[p] = make_float2(0.f, 0.f);
                    if (!rn) {
#pragma unroll
                        for (int r = 0; r < RPT; ++r) {
                            const int sl = M::row(warp, lane, r);
                            const float4 c = sm.ak[(t - 1) & 1][sl];
                            const float4 kq = sm.kq[sl];
                            const float2 ka = make_float2(c.x, c.y);
                            const float2 kap = make_float2(kq.x, kq.y), lam = make_float2(kq.z, kq.w);
#pragma unroll
                            for (int p = 0; p < 4; ++p) {
                                Z[r][p] = fma2(ka, ut[p], Z[r][p]);
                                pacc[p] = fma2(kap, Z[r][p], pacc[p]);
                                oacc[p] = fma2(lam, Z[r][p], oacc[p]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < RPT; ++r) {
                            const int sl = M::row(warp, lane, r);
                            const float4 c = sm.ak[(t - 1) & 1][sl];
                            const float4 kq = sm.kq[sl];
                            const float sr = sm.ak[t & 1][sl].w;
                            const float2 ka = make_float2(c.x, c.y), s2 = make_float2(sr, sr);
                            const float2 kap = make_float2(kq.x, kq.y), lam = make_float2(kq.z, kq.w);
#pragma unroll
                            for (int p = 0; p < 4; ++p) {
                                Z[r][p] = mul2(fma2(ka, ut[p], Z[r][p]), s2);
                                pacc[p] = fma2(kap, Z[r][p], pacc[p]);
                                oacc[p] = fma2(lam, Z[r][p], oacc[p]);
                            }
                        }
                    }
                    store_col_partials<D>(sm.red[warp][0], lane, pacc);
                    store_col_partials<D>(sm.red[warp][1], lane, oacc);
                }
                __syncthreads();
                if (tid < D) {   // u_t and o_t, column j
                    const int j = tid;
                    float ps = 0.f, os = 0.f, qk = 0.f;
#pragma unroll
                    for (int w = 0; w < M::kWarps; ++w) {
                        ps += sm.red[w][0][j];
                        os += sm.red[w][1][j];
                    }
#pragma unroll
                    for (int w = 0; w < D / 32; ++w) qk += sm.qkp[t & 1][w];
                    const float cj = sm.colc[j];
                    const float u = colA.beta * (colA.v - cj * ps);
                    a.o[(t * T + tile) * D + j] = fmaf(cj, os, qk * u);
                    sm.colb[j] = u * rcp_approx(cj);
                    if (t + 1 < a.chunk) colA.load(a, T, tile, j, t + 1);
                } else if (t + 1 < a.chunk) {   // meanwhile token t+1's constants
                    token_constants<D>(sm, he, tid - D, t + 1, rowA);
                    if (t + 2 < a.chunk) rowA.load(a, T, tile, tid - D, t + 2);
                }
                __syncthreads();
            }
            kb = (a.chunk - 1) & 1;
        }

        // ---- phase 3: X = D S + k u^T as alpha_i c_j Y_ij, Y = z + (k_i/alpha_i) u_j/c_j;
        //      row sums of |X| -------------------------------------------------------------
        if constexpr (kSplit) {
            float2 cf[4], ut[4];
            load_cols8(sm.colc, cl, cf);
            load_cols8(sm.colb, cl, ut);
            {
                // X_ij = alpha_i c_j Y_ij, written row by row in natural key order.
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int sl = M::row(warp, lane, r);
                    const float4 c = sm.ak[0][sl];
                    const float2 ka = make_float2(c.x, c.y), al = make_float2(c.z, c.z);
                    float4* dst = reinterpret_cast<float4*>(
                        a.x_out + (static_cast<int64_t>(tile) * D + (meta[sl] & 0xFF)) * D + 8 * cl);
                    float2 x[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) x[p] = mul2(mul2(fma2(ka, ut[p], Z[r][p]), al), cf[p]);
                    dst[0] = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
                    dst[1] = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
                }
                if (issued) {
                    sm.stage[sa].beta = next_beta;
                    sm.stage[sa].gate1 = next_gate;
                }
                __syncthreads();   // the next tile's prologue rewrites the per-slot constants
                continue;
            }
        }
        refit_pack<D, kPiv, true, kW>(sm, meta, Z, ww, kb, tile, a.r_out, a.c_out, a.packed_out + tile_base);
        if (issued) {   // ordered before their use by the barriers of the next tiles
            sm.stage[sa].beta = next_beta;
            sm.stage[sa].gate1 = next_gate;
        }
    }
}

// kSplit: the first kernel of the split form. It reconstructs, updates and reads out like the
// fused step, then writes the updated state X in fp32 and stops; the refit and the pack run
// as separate kernels (stepq_decode_step_split). kW: the row widths of a mixed launch's
// per-row code (a bit mask; 0 = every width).
template <int D, bool kSplit, bool kPiv, bool kChunk = false, bool kMixed = false, int kW = 0>
__global__ void __launch_bounds__(DMap<D>::kThreads, DMap<D>::kMinBlocks)
decode_kernel(const DecodeArgs a) {
    using M = DMap<D>;
    constexpr int RPT = M::RPT;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem<D>& sm = *reinterpret_cast<DecodeSmem<D>*>(smem_raw);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);
    // The last thread queues the copies (no prologue work waits on it).
    const bool issuer = (tid == M::kThreads - 1);

    // The first tiles' copies go out before anything else, so the HBM latency overlaps the
    // per-head table set-up.
    constexpr int CH = HeadCache<D>::kHeads;
    if (issuer) {
        for (int i = 0; i < kStages; ++i) mbar_init(&sm.full[i], 1);
        fence_barrier_init();
        for (int i = 0; i + 1 < kStages; ++i) {
            float b0, g0;
            if (issue_tile<D>(a, sm, cta_tile(i), i, b0, g0)) {
                sm.stage[i].beta = b0;
                sm.stage[i].gate1 = g0;
            }
        }
    }
    // Per-head tables (the bit map is frozen and shared by all sequences): the heads of the
    // CTA's first tiles are sorted up front, one warp per head; the rest on first use.
    for (int e = tid; e < CH; e += M::kThreads) sm.htag[e] = -1;
    __syncthreads();
    for (int n = warp; n < CH; n += M::kWarps) {
        const int tile = cta_tile(n);
        if (tile >= a.num_tiles) break;
        const int h = tile % a.H;
        // Sort here only if no earlier tile of this CTA uses the same head or the same entry.
        bool take = true;
        for (int m = 0; m < n; ++m)
            if ((cta_tile(m) % a.H) % CH == h % CH) take = false;
        if (take) {
            const int tot = sort_head_rows<D, kPiv>(a.bits + static_cast<int64_t>(h) * D, sm.hmeta[h % CH],
                                                    sm.hslot[h % CH], lane, &g_stepq_flags);
            if (lane == 0) {
                int64_t ho, hn;
                sm.hok[h % CH] = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, tot, 2 * D * D, &g_stepq_flags, &ho, &hn);
                sm.hoff[h % CH] = ho;
                sm.htag[h % CH] = h;
            }
        }
    }
    __syncthreads();

    run_tiles<D, kSplit, kPiv, kChunk, kMixed, kW>(a, sm);
}

template <int D, bool kSplit, bool kPiv, bool kChunk = false, bool kMixed = false, int kW = 0>
static int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(DecodeSmem<D>);
    if (a.num_tiles == 0) return STEPQ_OK;
    int grid = 0;
    int rc = persistent_grid(reinterpret_cast<const void*>(decode_kernel<D, kSplit, kPiv, kChunk, kMixed, kW>),
                             DMap<D>::kThreads, smem, a.num_tiles, "stepq_decode_step", &grid);
    if (rc) return rc;
    decode_kernel<D, kSplit, kPiv, kChunk, kMixed, kW><<<grid, DMap<D>::kThreads, smem, stream>>>(a);
    return check_launch("stepq_decode_step");
}

int device_flags_ptr(uint32_t** p) {
    static std::mutex mu;
    static uint32_t* ptrs[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(STEPQ_ECUDA, "device error word: device %d: %s", dev, cudaGetErrorString(e));
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptrs[dev]), g_stepq_flags);
        if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "device error word: %s", cudaGetErrorString(e));
    }
    *p = ptrs[dev];
    return STEPQ_OK;
}

// One event per device orders the refit and pack of the split form after its first kernel.
static int split_event(cudaEvent_t* ev) {
    static std::mutex mu;
    static cudaEvent_t events[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(STEPQ_ECUDA, "stepq_decode_step_split: device %d: %s", dev, cudaGetErrorString(e));
    std::lock_guard<std::mutex> lock(mu);
    if (events[dev] == nullptr) {
        e = cudaEventCreateWithFlags(&events[dev], cudaEventDisableTiming);
        if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "stepq_decode_step_split: %s", cudaGetErrorString(e));
    }
    *ev = events[dev];
    return STEPQ_OK;
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
    if (dims.widths & ~((1 << 2) | (1 << 4) | (1 << 6) | (1 << 8) | (1 << 16)))
        return set_error(STEPQ_EINVAL, "stepq_decode_step: widths=0x%x (bits 2, 4, 6, 8 and 16 only)", dims.widths);
    const long long tiles = static_cast<long long>(dims.B) * dims.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "stepq_decode_step: too many tiles");
    DecodeArgs a{dims.B, dims.H, dims.gate_per_channel, static_cast<int>(tiles), q, k, v, beta, gate, bits, w,
                 head_off, bytes_per_seq, packed_in, r_in, c_in, packed_out, r_out, c_out, o, nullptr, 1};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.mixed) {   // heads whose key rows have different widths: one code path for every width
        constexpr int W248 = (1 << 2) | (1 << 4) | (1 << 8), W468 = (1 << 4) | (1 << 6) | (1 << 8);
        const int wi = dims.widths & ~(1 << 16);   // the integer widths declared
        if (dims.dk == 128 && dims.widths != 0 && (wi & ~W248) == 0)
            return dims.pivots ? launch_decode<128, false, true, false, true, W248>(a, st)
                               : launch_decode<128, false, false, false, true, W248>(a, st);
        if (dims.dk == 128 && dims.widths != 0 && (wi & ~W468) == 0)
            return dims.pivots ? launch_decode<128, false, true, false, true, W468>(a, st)
                               : launch_decode<128, false, false, false, true, W468>(a, st);
        if (dims.pivots)
            return dims.dk == 128 ? launch_decode<128, false, true, false, true>(a, st)
                                  : launch_decode<64, false, true, false, true>(a, st);
        return dims.dk == 128 ? launch_decode<128, false, false, false, true>(a, st)
                              : launch_decode<64, false, false, false, true>(a, st);
    }
    if (dims.pivots) return dims.dk == 128 ? launch_decode<128, false, true>(a, st) : launch_decode<64, false, true>(a, st);
    return dims.dk == 128 ? launch_decode<128, false, false>(a, st) : launch_decode<64, false, false>(a, st);
}

extern "C" int stepq_prefill_chunk_seq(stepq_dims dims, int chunk, const uint16_t* q, const uint16_t* k,
                                       const uint16_t* v, const float* beta, const float* gate, const uint8_t* bits,
                                       const float* w, const int64_t* head_off, int64_t bytes_per_seq,
                                       const uint8_t* packed_in, const uint16_t* r_in, const uint16_t* c_in,
                                       uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out, float* o, void* stream) {
    const char* fn = "stepq_prefill_chunk_seq";
    clear_error();
    int rc = check_dims(dims, fn);
    if (rc) return rc;
    if (chunk < 1) return set_error(STEPQ_EINVAL, "%s: chunk=%d", fn, chunk);
    if (dims.B == 0) return STEPQ_OK;
    rc = check_ptrs(fn, {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate}, {"bits", bits}, {"w", w},
                         {"head_off", head_off}, {"packed_in", packed_in}, {"r_in", r_in}, {"c_in", c_in},
                         {"packed_out", packed_out}, {"r_out", r_out}, {"c_out", c_out}, {"o", o}});
    if (rc) return rc;
    if (bytes_per_seq <= 0 || (bytes_per_seq & 15))
        return set_error(STEPQ_EINVAL, "%s: bytes_per_seq=%lld", fn, (long long)bytes_per_seq);
    const long long tiles = static_cast<long long>(dims.B) * dims.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "%s: too many tiles", fn);
    DecodeArgs a{dims.B, dims.H, dims.gate_per_channel, static_cast<int>(tiles), q, k, v, beta, gate, bits, w,
                 head_off, bytes_per_seq, packed_in, r_in, c_in, packed_out, r_out, c_out, o, nullptr, chunk};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.mixed) {   // heads whose key rows have different widths: one code path for every width
        if (dims.pivots)
            return dims.dk == 128 ? launch_decode<128, false, true, true, true>(a, st)
                                  : launch_decode<64, false, true, true, true>(a, st);
        return dims.dk == 128 ? launch_decode<128, false, false, true, true>(a, st)
                              : launch_decode<64, false, false, true, true>(a, st);
    }
    if (dims.pivots)
        return dims.dk == 128 ? launch_decode<128, false, true, true>(a, st) : launch_decode<64, false, true, true>(a, st);
    return dims.dk == 128 ? launch_decode<128, false, false, true>(a, st) : launch_decode<64, false, false, true>(a, st);
}

extern "C" int stepq_decode_step_split(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                       const float* beta, const float* gate, const uint8_t* bits, const float* w,
                                       const int64_t* head_off, int64_t bytes_per_seq, const uint8_t* packed_in,
                                       const uint16_t* r_in, const uint16_t* c_in, uint8_t* packed_out,
                                       uint16_t* r_out, uint16_t* c_out, float* o, float* x_ws, void* stream,
                                       void* side_stream) {
    const char* fn = "stepq_decode_step_split";
    clear_error();
    int rc = check_dims(dims, fn);
    if (rc) return rc;
    if (dims.B == 0) return STEPQ_OK;
    rc = check_ptrs(fn, {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate}, {"bits", bits}, {"w", w},
                         {"head_off", head_off}, {"packed_in", packed_in}, {"r_in", r_in}, {"c_in", c_in},
                         {"o", o}, {"x_ws", x_ws}});
    if (rc) return rc;
    const bool refit = packed_out || r_out || c_out;
    if (refit) {
        rc = check_ptrs(fn, {{"packed_out", packed_out}, {"r_out", r_out}, {"c_out", c_out}});
        if (rc) return rc;
    }
    if (bytes_per_seq <= 0 || (bytes_per_seq & 15))
        return set_error(STEPQ_EINVAL, "%s: bytes_per_seq=%lld", fn, (long long)bytes_per_seq);
    const long long tiles = static_cast<long long>(dims.B) * dims.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "%s: too many tiles", fn);
    DecodeArgs a{dims.B, dims.H, dims.gate_per_channel, static_cast<int>(tiles), q, k, v, beta, gate, bits, w,
                 head_off, bytes_per_seq, packed_in, r_in, c_in, nullptr, nullptr, nullptr, o, x_ws, 1};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.pivots) rc = dims.dk == 128 ? launch_decode<128, true, true>(a, st) : launch_decode<64, true, true>(a, st);
    else rc = dims.dk == 128 ? launch_decode<128, true, false>(a, st) : launch_decode<64, true, false>(a, st);
    if (rc || !refit) return rc;
    // Refit and pack on the side stream, after the first kernel.
    cudaStream_t side = static_cast<cudaStream_t>(side_stream);
    cudaEvent_t ev;
    rc = split_event(&ev);
    if (rc) return rc;
    cudaError_t e = cudaEventRecord(ev, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev, 0);
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
    stepq_dims fd{dims.B, dims.H, dims.dk, dims.dv, 0, dims.pivots, 0};
    rc = stepq_fit_scales(fd, x_ws, w, bits, r_out, c_out, side_stream);
    if (rc) return rc;
    return stepq_pack_state(fd, x_ws, bits, head_off, bytes_per_seq, r_out, c_out, packed_out, side_stream);
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
