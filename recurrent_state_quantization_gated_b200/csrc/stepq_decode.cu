// stepq_decode.cu -- the fused quantized decode step (STEPQuant, Table C2) for sm_100a.
//
// One persistent CTA per SM slot walks over (sequence, head) tiles. For each tile the bulk-copy
// (TMA) engine stages the packed codes, the old scales, q/k/v, the gate and the head's bit map
// and row-impact vector into shared memory, double buffered so that the next tile's copy runs
// while this one is computed. The tile then lives in registers (a thread owns 4 columns of
// RPT rows) through every phase:
//   1 unpack + dequantise (the column scale is factored out: Xi_ij = X_ij / c_j), and the two
//     column dot products k^T X and q^T X of the Delta rule;
//   2 u = beta (v - k^T D S), o = q^T X = q^T D S + (q.k) u          (§2.1, Table C2 step 3);
//   3 X = D S + k u^T and the row factors m_i = mean_j |X_ij|        (§4.3 "Row factors");
//   4 the no-clip column initialisation c0_j                         (fit start);
//   5 codes at (r, c0) and the weighted least-squares column update   (App. C.1);
//   6 final codes at (r, c), packed and stored straight to HBM.
// Column reductions cross warps through shared memory; row reductions stay inside a warp.
// The state is read once and written once; no tensor cores (a rank-1 update per token is not
// a dense contraction).
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
    alignas(16) float4 rowc[D];     // alpha_i = g_i r_i 2^(8-b_i), alpha k_i, alpha q_i, k_i
    alignas(16) float4 rowq[D];     // 1/(r~_i 2^(8-b_i)), 1/q_b, (w_i r~_i 2^(8-b_i))^2, -
    alignas(16) float colc[D];      // c_j (old column scale)
    alignas(16) float colb[D];      // per-phase column broadcast
    alignas(16) float col0[D];      // c0_j
    alignas(16) float red[M::kWarps][2][D];
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
    alignas(16) uint16_t roff[D];
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
    uint32_t total = pbytes + 5u * 2u * D + D + 4u * D + (a.gate_per_channel ? 4u * D : 0u);
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

        // ---- prologue: per-row constants, row offsets, q.k -----------------------------
        if (tid < D) {
            const int i = tid;
            const int bw = st.bits[i];
            const float g = a.gate_per_channel ? st.gate[i] : __ldg(a.gate + tile);
            const float alpha = g * half_bits_to_float(st.r[i]) * znorm_of(bw);
            const float kk = bf16_bits_to_float(st.k[i]);
            const float qq = bf16_bits_to_float(st.q[i]);
            sm.rowc[i] = make_float4(alpha, alpha * kk, alpha * qq, kk);
        } else if (warp == D / 32) {
            row_offsets_warp<D>(st.bits, sm.roff, lane);
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

        // ---- phase 1: unpack, k^T X' and q^T X' (column scale factored out) ------------
        float Z[RPT][4];
        float pacc[4] = {0.f, 0.f, 0.f, 0.f}, oacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = M::row(warp, lane, r);
            const float4 rc = sm.rowc[i];
            unpack4<D>(st.codes + sm.roff[i], cl, st.bits[i], Z[r]);
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                pacc[kx] = fmaf(rc.y, Z[r][kx], pacc[kx]);
                oacc[kx] = fmaf(rc.z, Z[r][kx], oacc[kx]);
            }
        }
#pragma unroll
        for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                pacc[kx] += __shfl_xor_sync(0xffffffffu, pacc[kx], m);
                oacc[kx] += __shfl_xor_sync(0xffffffffu, oacc[kx], m);
            }
        if (lane < LPR) {
            *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(pacc[0], pacc[1], pacc[2], pacc[3]);
            *reinterpret_cast<float4*>(&sm.red[warp][1][4 * cl]) = make_float4(oacc[0], oacc[1], oacc[2], oacc[3]);
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

        // ---- phase 3: X = D S + k u^T (still divided by c_j), row |.| sums ------------
        float cf[4], ut[4];
        {
            const float4 c4 = *reinterpret_cast<const float4*>(&sm.colc[4 * cl]);
            const float4 u4 = *reinterpret_cast<const float4*>(&sm.colb[4 * cl]);
            cf[0] = c4.x; cf[1] = c4.y; cf[2] = c4.z; cf[3] = c4.w;
            ut[0] = u4.x; ut[1] = u4.y; ut[2] = u4.z; ut[3] = u4.w;
        }
        float part[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = M::row(warp, lane, r);
            const float4 rc = sm.rowc[i];
            float acc = 0.f;
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                const float x = fmaf(rc.x, Z[r][kx], rc.w * ut[kx]);
                Z[r][kx] = x;
                acc = fmaf(fabsf(x), cf[kx], acc);
            }
            part[r] = acc;
        }
        {
            int slot;
            bool owner;
            const float rsum = row_reduce<D, float>(sm.rowbuf[warp], lane, part, slot, OpAdd());
            const int i = reduced_row<D>(warp, lane, slot, owner);
            if (owner) {
                const int bw = st.bits[i];
                const float wi = st.w[i];
                const float m = rsum * (1.0f / D);
                const __half rh = scale_to_half(fmaxf(m, kHalfMinNormal) / wi);
                a.r_out[static_cast<int64_t>(tile) * D + i] = __half_as_ushort(rh);
                const float rs = __half2float(rh) * znorm_of(bw);
                const float g = wi * rs;
                sm.rowq[i] = make_float4(__frcp_rn(rs), __frcp_rn(static_cast<float>(qmax_of(bw))), g * g, 0.f);
            }
            __syncwarp();
        }

        // ---- phase 4: xi = X / (c_j r~_i 2^(8-b_i)); column no-clip scale c0 -----------
        float cmax[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = M::row(warp, lane, r);
            const float4 rq = sm.rowq[i];
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                const float x = Z[r][kx] * rq.x;
                Z[r][kx] = x;
                cmax[kx] = fmaxf(cmax[kx], fabsf(x) * rq.y);
            }
        }
#pragma unroll
        for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) cmax[kx] = fmaxf(cmax[kx], __shfl_xor_sync(0xffffffffu, cmax[kx], m));
        if (lane < LPR)
            *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(cmax[0], cmax[1], cmax[2], cmax[3]);
        __syncthreads();
        if (tid < D) {
            const int j = tid;
            float cm = 0.f;
#pragma unroll
            for (int w = 0; w < M::kWarps; ++w) cm = fmaxf(cm, sm.red[w][0][j]);
            const float cj = sm.colc[j];
            const float c0 = fmaxf(cj * cm, kHalfMinNormal);
            sm.col0[j] = c0;
            sm.colb[j] = cj / c0;
        }
        __syncthreads();

        // ---- phase 5: codes at (r~, c0); weighted least-squares column update ----------
        float f[4];
        {
            const float4 f4 = *reinterpret_cast<const float4*>(&sm.colb[4 * cl]);
            f[0] = f4.x; f[1] = f4.y; f[2] = f4.z; f[3] = f4.w;
        }
        float num[4] = {0.f, 0.f, 0.f, 0.f}, den[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = M::row(warp, lane, r);
            const float G = sm.rowq[i].z;
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                const float z0 = fmaf(Z[r][kx], f[kx], kRoundMagic) - kRoundMagic;
                const float gz = G * z0;
                num[kx] = fmaf(gz, Z[r][kx], num[kx]);
                den[kx] = fmaf(gz, z0, den[kx]);
            }
        }
#pragma unroll
        for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                num[kx] += __shfl_xor_sync(0xffffffffu, num[kx], m);
                den[kx] += __shfl_xor_sync(0xffffffffu, den[kx], m);
            }
        if (lane < LPR) {
            *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(num[0], num[1], num[2], num[3]);
            *reinterpret_cast<float4*>(&sm.red[warp][1][4 * cl]) = make_float4(den[0], den[1], den[2], den[3]);
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
            const float c1 = ds > 0.f ? (cj * ns) / ds : sm.col0[j];
            const __half ch = scale_to_half(c1);
            a.c_out[static_cast<int64_t>(tile) * D + j] = __half_as_ushort(ch);
            sm.colb[j] = cj / __half2float(ch);
        }
        __syncthreads();

        // ---- phase 6: final codes at (r~, c~), packed and stored -----------------------
        {
            const float4 f4 = *reinterpret_cast<const float4*>(&sm.colb[4 * cl]);
            f[0] = f4.x; f[1] = f4.y; f[2] = f4.z; f[3] = f4.w;
        }
        uint8_t* out = a.packed_out + tile_base;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = M::row(warp, lane, r);
            const int bw = st.bits[i];
            const int qb = qmax_of(bw);
            int qv[4];
#pragma unroll
            for (int kx = 0; kx < 4; ++kx) {
                const int t = __float_as_int(fmaf(Z[r][kx], f[kx], kRoundMagic)) - static_cast<int>(kRoundMagicBits);
                qv[kx] = min(max(t, -qb), qb);
            }
            pack4_store<D>(out + sm.roff[i], cl, bw, qv);
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
