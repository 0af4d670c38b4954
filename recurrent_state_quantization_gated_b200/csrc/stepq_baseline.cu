// stepq_baseline.cu -- the two comparison state formats of STEPQuant §5.1 on sm_100a: the FP32
// state (the serving default) and the quantisation of a state into the uniform symmetric
// rowwise-absmax INT8 format (its decode step is the persistent kernel of stepq_int8.cu), and the
// per-window 8-bit state. The decode steps take the readout before any requantisation.
//
// One CTA per (sequence, head) tile with the register mapping of stepq_device.cuh; the tile is
// loaded with 16-byte vector loads straight from HBM (each warp instruction reads one full row)
// and written back the same way.
#include <cuda_runtime.h>

#include "stepq_device.cuh"
#include "stepq_internal.h"

namespace stepq {

struct BaselineArgs {
    int H, gate_per_channel;
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* beta;
    const float* gate;
    const float* S_in;
    float* S_out;
    const int8_t* codes_in;
    const uint16_t* s_in;
    int8_t* codes_out;
    uint16_t* s_out;
    float* o;
};

template <int D>
struct BaselineSmem {
    using M = Map<D>;
    alignas(16) float4 rowc[D];     // alpha_i (gate x row scale), alpha k_i, alpha q_i, k_i
    alignas(16) float colu[D];
    alignas(16) float red[M::kWarps][2][D];
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
    alignas(16) float rows[D];      // int8: 1/s~_i
    float qk;
};

// Per-row constants (alpha_i = gate_i * row_scale_i) and q.k; one __syncthreads inside.
template <int D>
__device__ __forceinline__ void baseline_prologue(BaselineSmem<D>& sm, const BaselineArgs& a, int tile,
                                                  const uint16_t* row_scale) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < D) {
        const float g = a.gate_per_channel ? a.gate[static_cast<int64_t>(tile) * D + tid] : __ldg(a.gate + tile);
        const float sc = row_scale ? half_bits_to_float(row_scale[static_cast<int64_t>(tile) * D + tid]) : 1.0f;
        const float alpha = g * sc;
        const float kk = bf16_bits_to_float(a.k[static_cast<int64_t>(tile) * D + tid]);
        const float qq = bf16_bits_to_float(a.q[static_cast<int64_t>(tile) * D + tid]);
        sm.rowc[tid] = make_float4(alpha, alpha * kk, alpha * qq, kk);
    } else if (warp == D / 32) {
        constexpr int RL = D / 32;
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < RL; ++r) {
            const int i = lane * RL + r;
            acc = fmaf(bf16_bits_to_float(a.q[static_cast<int64_t>(tile) * D + i]),
                       bf16_bits_to_float(a.k[static_cast<int64_t>(tile) * D + i]), acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) sm.qk = acc;
    }
    __syncthreads();
}

// Shared middle of both kernels: Z holds the state divided by nothing (fp32) or the codes
// (int8) so that X_ij = alpha_i Z_ij before the update. Computes u and o, then overwrites Z
// with the updated state X = alpha Z + k u^T.
template <int D>
__device__ __forceinline__ void baseline_update(BaselineSmem<D>& sm, const BaselineArgs& a, int tile,
                                                float Z[Map<D>::RPT][4]) {
    using M = Map<D>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = M::col_lane(lane);
    float pacc[4] = {0.f, 0.f, 0.f, 0.f}, oacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const float4 rc = sm.rowc[M::row(warp, lane, r)];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            pacc[k] = fmaf(rc.y, Z[r][k], pacc[k]);
            oacc[k] = fmaf(rc.z, Z[r][k], oacc[k]);
        }
    }
    combine_subrows<Map<D>, float>(pacc, OpAdd());
    combine_subrows<Map<D>, float>(oacc, OpAdd());
    if (lane < M::LPR) {
        *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(pacc[0], pacc[1], pacc[2], pacc[3]);
        *reinterpret_cast<float4*>(&sm.red[warp][1][4 * cl]) = make_float4(oacc[0], oacc[1], oacc[2], oacc[3]);
    }
    __syncthreads();
    if (tid < D) {
        float ps = 0.f, os = 0.f;
#pragma unroll
        for (int w = 0; w < M::kWarps; ++w) {
            ps += sm.red[w][0][tid];
            os += sm.red[w][1][tid];
        }
        const float u = __ldg(a.beta + tile) * (bf16_bits_to_float(a.v[static_cast<int64_t>(tile) * D + tid]) - ps);
        a.o[static_cast<int64_t>(tile) * D + tid] = fmaf(sm.qk, u, os);
        sm.colu[tid] = u;
    }
    __syncthreads();
    const float4 u4 = *reinterpret_cast<const float4*>(&sm.colu[4 * cl]);
    const float u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const float4 rc = sm.rowc[M::row(warp, lane, r)];
#pragma unroll
        for (int k = 0; k < 4; ++k) Z[r][k] = fmaf(rc.x, Z[r][k], rc.w * u[k]);
    }
}

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads, Map<D>::kMinBlocks) decode_fp32_kernel(const BaselineArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    BaselineSmem<D>& sm = *reinterpret_cast<BaselineSmem<D>*>(smem_raw);
    const int tile = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = M::col_lane(lane);
    const float* S = a.S_in + static_cast<int64_t>(tile) * D * D;
    float Z[M::RPT][4];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(S + M::row(warp, lane, r) * D + 4 * cl));
        Z[r][0] = x.x; Z[r][1] = x.y; Z[r][2] = x.z; Z[r][3] = x.w;
    }
    baseline_prologue<D>(sm, a, tile, nullptr);
    baseline_update<D>(sm, a, tile, Z);
    float* So = a.S_out + static_cast<int64_t>(tile) * D * D;
#pragma unroll
    for (int r = 0; r < M::RPT; ++r)
        *reinterpret_cast<float4*>(So + M::row(warp, lane, r) * D + 4 * cl) = make_float4(Z[r][0], Z[r][1], Z[r][2], Z[r][3]);
}

// Rowwise absmax requantisation of a register tile; writes codes and scales.
template <int D, class Sm>
__device__ __forceinline__ void int8_requantise(Sm& sm, const float X[Map<D>::RPT][4], int tile,
                                                int8_t* codes_out, uint16_t* s_out) {
    using M = Map<D>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = M::col_lane(lane);
    float part[M::RPT];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r)
        part[r] = fmaxf(fmaxf(fabsf(X[r][0]), fabsf(X[r][1])), fmaxf(fabsf(X[r][2]), fabsf(X[r][3])));
    int slot;
    bool owner;
    const float mx = row_reduce<Map<D>, float>(sm.rowbuf[warp], lane, part, slot, OpMax());
    const int i = reduced_row<Map<D>>(warp, lane, slot, owner);
    if (owner) {
        const __half sh = scale_to_half(mx / 127.0f);
        s_out[static_cast<int64_t>(tile) * D + i] = __half_as_ushort(sh);
        sm.rows[i] = 1.0f / __half2float(sh);
    }
    __syncwarp();
    int8_t* out = codes_out + static_cast<int64_t>(tile) * D * D;
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int row = M::row(warp, lane, r);
        const float is = sm.rows[row];
        int q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = min(max(static_cast<int>(rintf(__fmul_rn(X[r][k], is))), -127), 127);
        const uint32_t t01 = __byte_perm(q[0], q[1], 0x0040);
        const uint32_t t23 = __byte_perm(q[2], q[3], 0x0040);
        *reinterpret_cast<uint32_t*>(out + row * D + 4 * cl) = __byte_perm(t01, t23, 0x5410);
    }
}

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads) int8_quantize_kernel(const BaselineArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    BaselineSmem<D>& sm = *reinterpret_cast<BaselineSmem<D>*>(smem_raw);
    const int tile = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = M::col_lane(lane);
    const float* S = a.S_in + static_cast<int64_t>(tile) * D * D;
    float X[M::RPT][4];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(S + M::row(warp, lane, r) * D + 4 * cl));
        X[r][0] = x.x; X[r][1] = x.y; X[r][2] = x.z; X[r][3] = x.w;
    }
    int8_requantise<D>(sm, X, tile, a.codes_out, a.s_out);
}

// ---- the per-window 8-bit state (LeapQuant: quantise once per window, buffered updates) ------
// Per tile, with the window's running log2 gate product l_s and gamma_s = 2^l_s, the state after
// token s of the window is S_s = gamma_s S_hat + sum_{r<=s} (gamma_s / gamma_r) k_r u_r^T, so
// token t needs only the fixed INT8 state and the buffered k_r, u_r (r < t):
//   p_t = S_{t-1}^T k_t = gamma_{t-1} S_hat^T k_t + sum_{r<t} (gamma_{t-1}/gamma_r) (k_r.k_t) u_r
//   u_t = beta_t (v_t - g_t p_t)
//   o_t = S_t^T q_t = gamma_t S_hat^T q_t + sum_{r<t} (gamma_t/gamma_r) (k_r.q_t) u_r + (k_t.q_t) u_t.
// The window's last token forms S_W in registers and requantises it (rowwise absmax INT8).
constexpr int kLeapMaxWindow = 256;

__device__ __forceinline__ void leap_cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void leap_cp4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void leap_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void leap_cp_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
constexpr int kLeapBatch = 16;   // buffered tokens staged per pass of the window-end update
constexpr int kLeapStage = 64;   // buffered tokens staged in shared memory per pass of a token

struct LeapArgs {
    int H, window, t, num_tiles;
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* beta;
    const float* gate;
    int8_t* codes;
    uint16_t* s;
    uint16_t* kbuf;
    float* ubuf;
    float* lbuf;
    float* o;
};

template <int D>
struct LeapSmem {
    using M = Map<D>;
    alignas(16) float2 rowc[D];                    // s_i k_i, s_i q_i
    alignas(16) float red[M::kWarps][2][D];
    alignas(16) float dots[2][kLeapMaxWindow];     // (gamma_{t-1}/gamma_r) k_r.k_t, (gamma_t/gamma_r) k_r.q_t
    alignas(16) float colu[D];                     // u_t
    alignas(16) float rowbuf[M::kWarps][32 * (M::RPT + 1)];
    alignas(16) float rows[D];
    alignas(16) float kb[kLeapBatch][D];           // window end: buffered keys
    alignas(16) float ub[kLeapBatch][D];           // window end: (gamma_W/gamma_r) u_r
    alignas(16) float us[kLeapStage][D];           // buffered u_r, staged for the column sums
    alignas(16) uint16_t ks[kLeapStage][D];        // buffered k_r, staged for the dot products
    alignas(16) float lr[kLeapStage];              // their running log2 gate products
    float qk, lprev, lt;
};

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads, Map<D>::kMinBlocks) leap_step_kernel(const LeapArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    LeapSmem<D>& sm = *reinterpret_cast<LeapSmem<D>*>(smem_raw);
    const int tile = blockIdx.x, t = a.t;
    const int64_t T = a.num_tiles;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = M::col_lane(lane);
    // The first kLeapStage buffered tokens' keys, pseudo-values and log gates are fetched first,
    // together with the tile's codes, so that their latencies overlap (independent 16-byte and
    // 4-byte asynchronous copies into shared memory).
    const int nb0 = min(kLeapStage, t);
    for (int e = tid; e < nb0 * (D / 8); e += M::kThreads) {
        const int rb = e / (D / 8), c8 = e % (D / 8);
        leap_cp16(&sm.ks[rb][8 * c8], a.kbuf + (static_cast<int64_t>(rb) * T + tile) * D + 8 * c8);
    }
    for (int e = tid; e < nb0 * (D / 4); e += M::kThreads) {
        const int rb = e / (D / 4), c4 = e % (D / 4);
        leap_cp16(&sm.us[rb][4 * c4], a.ubuf + (static_cast<int64_t>(rb) * T + tile) * D + 4 * c4);
    }
    for (int e = tid; e < nb0; e += M::kThreads) leap_cp4(&sm.lr[e], a.lbuf + static_cast<int64_t>(e) * T + tile);
    leap_cp_commit();
    // This token's v_j, beta and gate for the final column step, fetched now as well.
    float vj = 0.f, bt = 0.f, gt = 0.f;
    if (tid < D) {
        vj = bf16_bits_to_float(__ldg(a.v + static_cast<int64_t>(tile) * D + tid));
        bt = __ldg(a.beta + tile);
        gt = __ldg(a.gate + tile);
    }
    const int8_t* Cd = a.codes + static_cast<int64_t>(tile) * D * D;
    float Z[M::RPT][4];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(Cd + M::row(warp, lane, r) * D + 4 * cl)) ^ 0x80808080u;
#pragma unroll
        for (int c = 0; c < 4; ++c) Z[r][c] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650 | c)) - (kTwo23 + 128.0f);
    }
    const uint16_t* kt_g = a.k + static_cast<int64_t>(tile) * D;
    const uint16_t* qt_g = a.q + static_cast<int64_t>(tile) * D;
    if (tid < D) {
        const float si = half_bits_to_float(a.s[static_cast<int64_t>(tile) * D + tid]);
        const uint16_t kb = kt_g[tid];
        sm.rowc[tid] = make_float2(si * bf16_bits_to_float(kb), si * bf16_bits_to_float(qt_g[tid]));
        a.kbuf[(static_cast<int64_t>(t) * T + tile) * D + tid] = kb;   // this token joins the window's buffer
    }
    if (tid == 0) {
        const float lp = t > 0 ? a.lbuf[static_cast<int64_t>(t - 1) * T + tile] : 0.0f;
        const float lt = lp + log2f(fmaxf(__ldg(a.gate + tile), 0x1p-64f));   // a zero gate counts 2^-64
        sm.lprev = lp;
        sm.lt = lt;
        a.lbuf[static_cast<int64_t>(t) * T + tile] = lt;
    }
    __syncthreads();
    // k_t and q_t of this lane's D/32 key rows, for the dot products with the buffered keys.
    constexpr int RL = D / 32;
    float kl[RL], ql[RL];
#pragma unroll
    for (int e = 0; e < RL; ++e) {
        kl[e] = bf16_bits_to_float(kt_g[lane * RL + e]);
        ql[e] = bf16_bits_to_float(qt_g[lane * RL + e]);
    }
    if (warp == 0) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < RL; ++e) acc = fmaf(kl[e], ql[e], acc);
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        if (lane == 0) sm.qk = acc;
    }
    leap_cp_wait();
    __syncthreads();
    // The buffered tokens' dot products with k_t and q_t, kLeapStage tokens at a time (the first
    // stage is already in shared memory; later ones are staged with independent 16-byte loads),
    // one warp per buffered token.
    for (int r0 = 0; r0 < t; r0 += kLeapStage) {
        const int nb = min(kLeapStage, t - r0);
        if (r0 > 0) {
            for (int e = tid; e < nb * (D / 8); e += M::kThreads) {
                const int rb = e / (D / 8), c8 = e % (D / 8);
                *reinterpret_cast<uint4*>(&sm.ks[rb][8 * c8]) = __ldg(reinterpret_cast<const uint4*>(
                    a.kbuf + (static_cast<int64_t>(r0 + rb) * T + tile) * D + 8 * c8));
            }
            __syncthreads();
        }
        for (int rb = warp; rb < nb; rb += M::kWarps) {
            float ck = 0.f, cq = 0.f;
#pragma unroll
            for (int e = 0; e < RL; ++e) {
                const float x = bf16_bits_to_float(sm.ks[rb][lane * RL + e]);
                ck = fmaf(x, kl[e], ck);
                cq = fmaf(x, ql[e], cq);
            }
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) {
                ck += __shfl_xor_sync(0xffffffffu, ck, m);
                cq += __shfl_xor_sync(0xffffffffu, cq, m);
            }
            if (lane == 0) {
                const float lr = r0 == 0 ? sm.lr[rb] : a.lbuf[static_cast<int64_t>(r0 + rb) * T + tile];
                sm.dots[0][r0 + rb] = ck * exp2f(sm.lprev - lr);
                sm.dots[1][r0 + rb] = cq * exp2f(sm.lt - lr);
            }
        }
        if (r0 + kLeapStage < t) __syncthreads();   // the next stage rewrites the keys
    }
    // S_hat^T k_t and S_hat^T q_t, column partial sums.
    {
        float pacc[4] = {0.f, 0.f, 0.f, 0.f}, oacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < M::RPT; ++r) {
            const float2 rc = sm.rowc[M::row(warp, lane, r)];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                pacc[c] = fmaf(rc.x, Z[r][c], pacc[c]);
                oacc[c] = fmaf(rc.y, Z[r][c], oacc[c]);
            }
        }
        combine_subrows<Map<D>, float>(pacc, OpAdd());
        combine_subrows<Map<D>, float>(oacc, OpAdd());
        if (lane < M::LPR) {
            *reinterpret_cast<float4*>(&sm.red[warp][0][4 * cl]) = make_float4(pacc[0], pacc[1], pacc[2], pacc[3]);
            *reinterpret_cast<float4*>(&sm.red[warp][1][4 * cl]) = make_float4(oacc[0], oacc[1], oacc[2], oacc[3]);
        }
    }
    __syncthreads();
    // The buffered u_r weighted by those dot products, kLeapStage tokens at a time (staged with
    // independent 16-byte loads); threads j < D own column j.
    float bp = 0.f, bo = 0.f;
    for (int r0 = 0; r0 < t; r0 += kLeapStage) {
        const int nb = min(kLeapStage, t - r0);
        if (r0 > 0) {   // the first stage was fetched at the start
            __syncthreads();   // the previous stage has been read
            for (int e = tid; e < nb * (D / 4); e += M::kThreads) {
                const int rb = e / (D / 4), c4 = e % (D / 4);
                *reinterpret_cast<float4*>(&sm.us[rb][4 * c4]) = __ldg(reinterpret_cast<const float4*>(
                    a.ubuf + (static_cast<int64_t>(r0 + rb) * T + tile) * D + 4 * c4));
            }
            __syncthreads();
        }
        if (tid < D) {
#pragma unroll 4
            for (int rb = 0; rb < nb; ++rb) {
                const float u = sm.us[rb][tid];
                bp = fmaf(sm.dots[0][r0 + rb], u, bp);
                bo = fmaf(sm.dots[1][r0 + rb], u, bo);
            }
        }
    }
    if (tid < D) {   // column j: u_t and o_t
        const int j = tid;
        float a0 = 0.f, b0 = 0.f;
#pragma unroll
        for (int w = 0; w < M::kWarps; ++w) {
            a0 += sm.red[w][0][j];
            b0 += sm.red[w][1][j];
        }
        const float p = fmaf(exp2f(sm.lprev), a0, bp);
        const float u = bt * (vj - gt * p);
        a.o[static_cast<int64_t>(tile) * D + j] = fmaf(sm.qk, u, fmaf(exp2f(sm.lt), b0, bo));
        a.ubuf[(static_cast<int64_t>(t) * T + tile) * D + j] = u;
        sm.colu[j] = u;
    }
    if (t + 1 < a.window) return;

    // ---- the window's last token: S_W = gamma_W S_hat + sum_r (gamma_W/gamma_r) k_r u_r^T ----
    __syncthreads();
    {
        const float gw = exp2f(sm.lt);
#pragma unroll
        for (int r = 0; r < M::RPT; ++r) {
            const float f = gw * half_bits_to_float(a.s[static_cast<int64_t>(tile) * D + M::row(warp, lane, r)]);
#pragma unroll
            for (int c = 0; c < 4; ++c) Z[r][c] *= f;
        }
    }
    for (int r0 = 0; r0 <= t; r0 += kLeapBatch) {
        const int nb = min(kLeapBatch, t + 1 - r0);
        __syncthreads();   // the previous batch has been used
        for (int e = tid; e < nb * D; e += M::kThreads) {
            const int rb = e / D, i = e % D, r = r0 + rb;
            sm.kb[rb][i] = bf16_bits_to_float(r == t ? kt_g[i] : a.kbuf[(static_cast<int64_t>(r) * T + tile) * D + i]);
            const float u = r == t ? sm.colu[i] : a.ubuf[(static_cast<int64_t>(r) * T + tile) * D + i];
            const float lr = r == t ? sm.lt : a.lbuf[static_cast<int64_t>(r) * T + tile];
            sm.ub[rb][i] = u * exp2f(sm.lt - lr);
        }
        __syncthreads();
        for (int rb = 0; rb < nb; ++rb) {
            const float4 u4 = *reinterpret_cast<const float4*>(&sm.ub[rb][4 * cl]);
#pragma unroll
            for (int r = 0; r < M::RPT; ++r) {
                const float kk = sm.kb[rb][M::row(warp, lane, r)];
                Z[r][0] = fmaf(kk, u4.x, Z[r][0]);
                Z[r][1] = fmaf(kk, u4.y, Z[r][1]);
                Z[r][2] = fmaf(kk, u4.z, Z[r][2]);
                Z[r][3] = fmaf(kk, u4.w, Z[r][3]);
            }
        }
    }
    __syncthreads();   // every thread has read its codes and the scales before they are rewritten
    int8_requantise<D>(sm, Z, tile, a.codes, a.s);
}

template <int D>
static int launch_baseline(const char* fn, void (*kern)(BaselineArgs), int tiles, const BaselineArgs& a,
                           cudaStream_t st) {
    if (tiles == 0) return STEPQ_OK;
    const size_t smem = sizeof(BaselineSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
    kern<<<tiles, Map<D>::kThreads, smem, st>>>(a);
    return check_launch(fn);
}

static int tiles_of(const stepq_dims& d, const char* fn, long long& tiles) {
    int rc = check_dims(d, fn);
    if (rc) return rc;
    tiles = static_cast<long long>(d.B) * d.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "%s: too many tiles", fn);
    return STEPQ_OK;
}

}  // namespace stepq

using namespace stepq;

extern "C" int stepq_decode_step_fp32(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                      const float* beta, const float* gate, const float* S_in, float* S_out,
                                      float* o, void* stream) {
    clear_error();
    long long tiles;
    int rc = tiles_of(dims, "stepq_decode_step_fp32", tiles);
    if (rc || tiles == 0) return rc;
    rc = check_ptrs("stepq_decode_step_fp32", {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate},
                                               {"S_in", S_in}, {"S_out", S_out}, {"o", o}});
    if (rc) return rc;
    BaselineArgs a{};
    a.H = dims.H; a.gate_per_channel = dims.gate_per_channel; a.q = q; a.k = k; a.v = v; a.beta = beta;
    a.gate = gate; a.S_in = S_in; a.S_out = S_out; a.o = o;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128 ? launch_baseline<128>("stepq_decode_step_fp32", decode_fp32_kernel<128>, (int)tiles, a, st)
                          : launch_baseline<64>("stepq_decode_step_fp32", decode_fp32_kernel<64>, (int)tiles, a, st);
}

extern "C" int stepq_int8_quantize_state(stepq_dims dims, const float* S, int8_t* codes, uint16_t* s, void* stream) {
    clear_error();
    long long tiles;
    int rc = tiles_of(dims, "stepq_int8_quantize_state", tiles);
    if (rc || tiles == 0) return rc;
    rc = check_ptrs("stepq_int8_quantize_state", {{"S", S}, {"codes", codes}, {"s", s}});
    if (rc) return rc;
    BaselineArgs a{};
    a.H = dims.H; a.S_in = S; a.codes_out = codes; a.s_out = s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128
               ? launch_baseline<128>("stepq_int8_quantize_state", int8_quantize_kernel<128>, (int)tiles, a, st)
               : launch_baseline<64>("stepq_int8_quantize_state", int8_quantize_kernel<64>, (int)tiles, a, st);
}

extern "C" int stepq_leap_step(stepq_dims dims, int window, int t, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const float* beta, const float* gate, int8_t* codes, uint16_t* s,
                               uint16_t* kbuf, float* ubuf, float* lbuf, float* o, void* stream) {
    const char* fn = "stepq_leap_step";
    clear_error();
    long long tiles;
    int rc = tiles_of(dims, fn, tiles);
    if (rc) return rc;
    if (dims.gate_per_channel)
        return set_error(STEPQ_EUNSUPPORTED, "%s: channel gates are not supported by the per-window form", fn);
    if (window < 1 || window > kLeapMaxWindow || t < 0 || t >= window)
        return set_error(STEPQ_EINVAL, "%s: window=%d t=%d (need 0 <= t < window <= %d)", fn, window, t, kLeapMaxWindow);
    if (tiles == 0) return STEPQ_OK;
    rc = check_ptrs(fn, {{"q", q}, {"k", k}, {"v", v}, {"beta", beta}, {"gate", gate}, {"codes", codes}, {"s", s},
                         {"kbuf", kbuf}, {"ubuf", ubuf}, {"lbuf", lbuf}, {"o", o}});
    if (rc) return rc;
    LeapArgs a{dims.H, window, t, static_cast<int>(tiles), q, k, v, beta, gate, codes, s, kbuf, ubuf, lbuf, o};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto go = [&](auto kern, size_t smem) -> int {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
        kern<<<static_cast<int>(tiles), dims.dk == 128 ? Map<128>::kThreads : Map<64>::kThreads, smem, st>>>(a);
        return check_launch(fn);
    };
    return dims.dk == 128 ? go(leap_step_kernel<128>, sizeof(LeapSmem<128>)) : go(leap_step_kernel<64>, sizeof(LeapSmem<64>));
}

namespace stepq {
// One bounded wait that nothing completes: a fresh mbarrier's phase 0 never sees an arrival, so
// the wait gives up after limit_ns and raises bit 0 of the device error word, as a stalled tile
// copy or tensor-core round would in the library's kernels.
__global__ void wait_selftest_kernel(uint64_t limit_ns, uint32_t* flags) {
    __shared__ alignas(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit_ns, flags);
}
}  // namespace stepq

extern "C" int stepq_selftest_wait(uint64_t limit_ns, void* stream) {
    clear_error();
    if (limit_ns < 1000 || limit_ns > 1000000000ull)
        return set_error(STEPQ_EINVAL, "stepq_selftest_wait: limit_ns=%llu (need 1e3 to 1e9)", (unsigned long long)limit_ns);
    uint32_t* flags = nullptr;
    int rc = device_flags_ptr(&flags);
    if (rc) return rc;
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, flags);
    return check_launch("stepq_selftest_wait");
}
