// stepq_int8.cu -- the decode step on the uniform symmetric rowwise-absmax INT8 state, the
// comparison format of STEPQuant §5.1, as a persistent kernel for sm_100a.
//
// Each CTA walks over (sequence, head) tiles. The bulk-copy (TMA) engine stages a tile's codes,
// row scales, q, k, v and gate into shared memory three tiles deep, so the next tiles' bytes
// arrive while this one is computed. The tile lives in registers (a thread owns 8 columns of
// D/16 rows) in the factored form X_ij = alpha_i Y_ij, alpha_i = g_i s_i:
//   1 codes -> floats (Y = z), the column dot products k^T D S and q^T D S;
//   2 u = beta (v - k^T D S) and the readout o = q^T X = q^T D S + (q.k) u     (§2.1);
//   3 Y += (k_i / alpha_i) u_j, the row maxima of |Y|, new row scales s~_i = fp16(alpha_i max/127);
//   4 codes rint(Y alpha_i / s~_i) limited to [-127, 127], written over the staged codes, and one
//     bulk store (TMA, 1-D) of the whole tile.
// The state is read once and written once; no tensor cores (a rank-1 update is not a contraction).
#include <cuda_runtime.h>

#include "stepq_device.cuh"
#include "stepq_internal.h"
#include "stepq_tile.cuh"

namespace stepq {
namespace {

constexpr int kI8Stages = 3;
constexpr uint64_t kI8WaitNs = 2000000000ull;   // 2 s: a tile copy takes microseconds

struct Int8Args {
    int H, gate_per_channel, num_tiles;
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* beta;
    const float* gate;
    const int8_t* codes_in;
    const uint16_t* s_in;
    int8_t* codes_out;
    uint16_t* s_out;
    float* o;
    uint32_t* flags;   // device error word (bit 0: a bounded wait gave up)
};

template <int D>
struct Int8Smem {
    using M = DMap<D>;
    struct Stage {
        alignas(128) int8_t codes[D * D];   // the tile's codes; the new codes are written over them
        alignas(16) uint16_t s[D];
        alignas(16) uint16_t q[D];
        alignas(16) uint16_t k[D];
        alignas(16) uint16_t v[D];
        alignas(16) float gate[D];
        float beta, gate1;
    };
    Stage stage[kI8Stages];
    alignas(16) float4 rowc[D];   // alpha k_i, alpha q_i, k_i / alpha, alpha    (alpha = g_i s_i)
    alignas(16) float rowq[D];    // alpha_i / s~_i: the requantisation factor of row i
    alignas(16) float colu[D];    // u_j
    alignas(16) float red[M::kWarps][2][M::kRedRow];
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
    float qkp[M::kWarps];
    alignas(8) uint64_t full[kI8Stages];
};

__device__ __forceinline__ int i8_tile(int n) { return blockIdx.x + n * gridDim.x; }

// The two scalars of a tile (beta, and the gate unless it is per channel), loaded by the issuing
// thread one tile before it queues the tile's copies, so that their latency stays hidden.
struct I8Scalars {
    float beta = 0.f, gate1 = 0.f;
};

__device__ __forceinline__ I8Scalars i8_scalars(const Int8Args& a, int tile) {
    I8Scalars t;
    if (tile < a.num_tiles) {
        t.beta = __ldg(a.beta + tile);
        t.gate1 = a.gate_per_channel ? 0.f : __ldg(a.gate + tile);
    }
    return t;
}

// Queues the bulk copies of `tile` into stage s and stores its scalars there (one thread).
template <int D>
__device__ __forceinline__ void i8_issue(const Int8Args& a, Int8Smem<D>& sm, int tile, int s, const I8Scalars& sc) {
    if (tile >= a.num_tiles) return;
    auto& st = sm.stage[s];
    const int64_t t = tile;
    const uint32_t bytes = D * D + 4u * 2u * D + (a.gate_per_channel ? 4u * D : 0u);
    mbar_arrive_expect_tx(&sm.full[s], bytes);
    bulk_load(st.codes, a.codes_in + t * D * D, D * D, &sm.full[s]);
    bulk_load(st.s, a.s_in + t * D, 2 * D, &sm.full[s]);
    bulk_load(st.q, a.q + t * D, 2 * D, &sm.full[s]);
    bulk_load(st.k, a.k + t * D, 2 * D, &sm.full[s]);
    bulk_load(st.v, a.v + t * D, 2 * D, &sm.full[s]);
    if (a.gate_per_channel) bulk_load(st.gate, a.gate + t * D, 4 * D, &sm.full[s]);
    st.beta = sc.beta;
    st.gate1 = sc.gate1;
}

template <int D>
__global__ void __launch_bounds__(DMap<D>::kThreads, DMap<D>::kMinBlocks) int8_step_kernel(const Int8Args a) {
    using M = DMap<D>;
    constexpr int RPT = M::RPT;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Int8Smem<D>& sm = *reinterpret_cast<Int8Smem<D>*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    const bool issuer = (tid == M::kThreads - 1);
    const float2 M2 = make_float2(kRoundMagic, kRoundMagic);

    if (issuer) {
        for (int i = 0; i < kI8Stages; ++i) mbar_init(&sm.full[i], 1);
        fence_barrier_init();
        for (int i = 0; i + 1 < kI8Stages; ++i) i8_issue<D>(a, sm, i8_tile(i), i, i8_scalars(a, i8_tile(i)));
    }
    __syncthreads();

    for (int n = 0;; ++n) {
        const int tile = i8_tile(n);
        if (tile >= a.num_tiles) break;
        const int s = n % kI8Stages;
        auto& st = sm.stage[s];
        const int ahead = n + kI8Stages - 1, sa = ahead % kI8Stages;
        I8Scalars next;
        if (issuer) next = i8_scalars(a, i8_tile(ahead));
        const bool ok = mbar_wait_bounded(&sm.full[s], (n / kI8Stages) & 1, kI8WaitNs, a.flags);
        if (__syncthreads_or(!ok)) {
            // A tile copy never arrived: give up after one more bounded wait for each copy in flight.
            if (issuer)
                for (int i = 1; i < kI8Stages; ++i)
                    if (i8_tile(n + i) < a.num_tiles)
                        mbar_wait_bounded(&sm.full[(n + i) % kI8Stages], ((n + i) / kI8Stages) & 1, kI8WaitNs,
                                          a.flags);
            break;
        }
        // Every thread is past the previous tile: the copies of the tile kI8Stages-1 ahead go into
        // its stage once the previous tile's bulk store has read it out.
        if (issuer) {
            bulk_wait_read_all();
            i8_issue<D>(a, sm, i8_tile(ahead), sa, next);
        }

        // ---- per-row constants of the warp's own rows, and its share of q.k ----------------
        {
            float qk = 0.f;
            if (lane < M::kRowsPerWarp) {
                const int i = warp * M::kRowsPerWarp + lane;
                const float g = a.gate_per_channel ? st.gate[i] : st.gate1;
                // alpha > 0 always (a zero gate leaves 2^-64, far below any term that counts)
                const float alpha = fmaxf(g * half_bits_to_float(st.s[i]), 0x1p-64f);
                const float kk = bf16_bits_to_float(st.k[i]), qq = bf16_bits_to_float(st.q[i]);
                sm.rowc[i] = make_float4(alpha * kk, alpha * qq, kk * rcp_approx(alpha), alpha);
                qk = qq * kk;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);
            if (lane == 0) sm.qkp[warp] = qk;
        }
        __syncwarp();

        // ---- 1: codes -> floats; k^T D S and q^T D S ------------------------------------
        float2 Z[RPT][4];
        {
            float2 pacc[4], oacc[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) pacc[p] = oacc[p] = make_float2(0.f, 0.f);
            uint2 raw[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r)
                raw[r] = *reinterpret_cast<const uint2*>(st.codes + M::row(warp, lane, r) * D + 8 * cl);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                unpack8r<8>(raw[r], Z[r]);
                const float4 c = sm.rowc[M::row(warp, lane, r)];
                const float2 ak = make_float2(c.x, c.x), aq = make_float2(c.y, c.y);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    pacc[p] = fma2(ak, Z[r][p], pacc[p]);
                    oacc[p] = fma2(aq, Z[r][p], oacc[p]);
                }
            }
            store_col_partials<D>(sm.red[warp][0], lane, pacc);
            store_col_partials<D>(sm.red[warp][1], lane, oacc);
        }
        __syncthreads();

        // ---- 2: u and the readout (threads < D, one column each); the copies of the tile
        //         kI8Stages-1 ahead go out meanwhile, into the stage of the previous tile -------
        {   // every thread: k^T D S (lanes 0-15) or q^T D S (16-31) of one column
            const int j = M::fin_col(warp, lane), qd = M::fin_row(lane);
            float acc = 0.f, qk = 0.f;
#pragma unroll
            for (int w = 0; w < M::kWarps; ++w) {
                acc += sm.red[w][qd][j];
                qk += sm.qkp[w];
            }
            const float oth = __shfl_xor_sync(0xffffffffu, acc, 16);
            if (qd == 0) {
                const float u = st.beta * (bf16_bits_to_float(st.v[j]) - acc);
                a.o[static_cast<int64_t>(tile) * D + j] = fmaf(qk, u, oth);
                sm.colu[j] = u;
            }
        }
        __syncthreads();

        // ---- 3: rank-1 update Y += (k_i/alpha_i) u_j; row maxima of |Y|; new row scales ------
        {
            float2 u2[4];
            load_cols8(sm.colu, cl, u2);
            float part[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float kap = sm.rowc[M::row(warp, lane, r)].z;
                const float2 k2 = make_float2(kap, kap);
#pragma unroll
                for (int p = 0; p < 4; ++p) Z[r][p] = fma2(k2, u2[p], Z[r][p]);
                float m = max_abs3(Z[r][0].x, Z[r][0].y, Z[r][1].x);
                m = max_abs3(m, Z[r][1].y, Z[r][2].x);
                m = max_abs3(m, Z[r][2].y, Z[r][3].x);
                part[r] = fmaxf(m, fabsf(Z[r][3].y));
            }
            int slot;
            bool owner;
            const float mx = row_reduce<M, float>(sm.rowbuf[warp], lane, part, slot, OpMax());
            const int i = reduced_row<M>(warp, lane, slot, owner);
            if (owner) {
                // X_ij = alpha_i Y_ij, alpha_i > 0: the row maximum of |X| is alpha_i max |Y|
                const float alpha = sm.rowc[i].w;
                const __half sh = scale_to_half(alpha * mx / 127.0f);
                a.s_out[static_cast<int64_t>(tile) * D + i] = __half_as_ushort(sh);
                sm.rowq[i] = alpha * (1.0f / __half2float(sh));
            }
            __syncwarp();
        }

        // ---- 4: codes rint(X / s~_i) in [-127, 127] over the staged codes, one bulk store ------
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = M::row(warp, lane, r);
            const float f = sm.rowq[i];
            const float2 f2 = make_float2(f, f);
            uint32_t zq[8];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 t = fma2(Z[r][p], f2, M2);
                zq[2 * p] = __float_as_uint(t.x);
                zq[2 * p + 1] = __float_as_uint(t.y);
            }
            *reinterpret_cast<uint2*>(st.codes + i * D + 8 * cl) =
                make_uint2(gather4<8, true>(zq[0], zq[1], zq[2], zq[3]), gather4<8, true>(zq[4], zq[5], zq[6], zq[7]));
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (issuer) {
            bulk_store(a.codes_out + static_cast<int64_t>(tile) * D * D, st.codes, D * D);
            bulk_commit();
        }
    }
    if (issuer) bulk_wait_all();
}

template <int D>
int launch_int8(const Int8Args& a, cudaStream_t st) {
    const char* fn = "stepq_decode_step_int8";
    int grid = 0;
    const size_t smem = sizeof(Int8Smem<D>);
    int rc = persistent_grid(reinterpret_cast<const void*>(int8_step_kernel<D>), DMap<D>::kThreads, smem,
                             a.num_tiles, fn, &grid);
    if (rc) return rc;
    int8_step_kernel<D><<<grid, DMap<D>::kThreads, smem, st>>>(a);
    return check_launch(fn);
}

}  // namespace
}  // namespace stepq

using namespace stepq;

extern "C" int stepq_decode_step_int8(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                      const float* beta, const float* gate, const int8_t* codes_in,
                                      const uint16_t* s_in, int8_t* codes_out, uint16_t* s_out, float* o,
                                      void* stream) {
    const char* fn = "stepq_decode_step_int8";
    clear_error();
    int rc = check_dims(dims, fn);
    if (rc) return rc;
    const long long tiles = static_cast<long long>(dims.B) * dims.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "%s: too many tiles", fn);
    if (tiles == 0) return STEPQ_OK;
    rc = check_ptrs(fn, {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate}, {"codes_in", codes_in},
                         {"s_in", s_in}, {"codes_out", codes_out}, {"s_out", s_out}, {"o", o}});
    if (rc) return rc;
    Int8Args a{dims.H, dims.gate_per_channel, static_cast<int>(tiles), q, k, v, beta, gate, codes_in, s_in,
               codes_out, s_out, o, nullptr};
    rc = device_flags_ptr(&a.flags);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128 ? launch_int8<128>(a, st) : launch_int8<64>(a, st);
}
