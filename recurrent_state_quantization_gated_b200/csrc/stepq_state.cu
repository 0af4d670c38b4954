// stepq_state.cu -- state conversion kernels of libstepq (sm_100a): the key-row-aware
// dual-axis fit (STEPQuant §4.3, App. C.1), packing with the quantisation contract (§2.2),
// unpacking with the dequantisation contract, and the candidate-format distortion used by the
// offline bit allocation (App. A.3, Eq. 17 / Eq. 18).
//
// One CTA per (sequence, head) tile, the tile held in registers with the mapping of
// stepq_device.cuh. These run once per state (or once per calibration), not per token, so the
// fit accumulates its reductions in float64: its scales then agree with a float64 reference
// up to the final binary16 rounding.
#include <cuda_runtime.h>

#include <mutex>

#include "stepq_device.cuh"
#include "stepq_internal.h"

namespace stepq {

template <int D>
struct TileSmem {
    using M = Map<D>;
    alignas(16) uint8_t bits[D];
    alignas(16) float w[D];
    alignas(16) float4 rowa[D];      // a_i, ir_i, w_i, r~_i 2^(8-b_i)
    alignas(16) float colf[D];       // 1/c0_j, later 1/c~_j
    alignas(16) float col0[D];
    alignas(16) float colc[D];       // c~_j
    alignas(16) double red[M::kWarps][2][D];
    alignas(16) double rowbuf[M::kWarps][32 * (M::RPT + 1)];
    alignas(16) uint16_t roff[D];
    int ok;                          // pack / unpack: the head's byte range holds the tile
};

// The quantisation contract: t = (x * ir) * ic, nearest-even, clamped to [-q_b, q_b].
__device__ __forceinline__ int quantise(float x, float ir, float ic, int qb) {
    const float t = __fmul_rn(__fmul_rn(x, ir), ic);
    const int n = static_cast<int>(rintf(t));
    return min(max(n, -qb), qb);
}

// Load the RPT x 4 entries this thread owns from a row-major fp32 tile.
template <int D>
__device__ __forceinline__ void load_tile(const float* S, int warp, int lane, float X[Map<D>::RPT][4]) {
    using M = Map<D>;
    const int cl = M::col_lane(lane);
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int i = M::row(warp, lane, r);
        const float4 x = __ldg(reinterpret_cast<const float4*>(S + i * D + 4 * cl));
        X[r][0] = x.x; X[r][1] = x.y; X[r][2] = x.z; X[r][3] = x.w;
    }
}

// The dual-axis fit of a register-resident tile. sm.bits and sm.w must be loaded (and a
// __syncthreads issued) before the call. Writes r (binary16 bits, [D]) and c ([D]) and leaves
// the scales in sm.rowa / sm.colc / sm.colf (= 1/c~) for a following quantisation.
template <int D>
__device__ void fit_tile_regs(TileSmem<D>& sm, const float X[Map<D>::RPT][4], int warp, int lane,
                              uint16_t* r_out, uint16_t* c_out) {
    using M = Map<D>;
    constexpr int RPT = M::RPT;
    const int tid = threadIdx.x;
    const int cl = M::col_lane(lane);

    // Row factors: m_i = mean_j |X_ij|; r_i = fp16(clamp(max(m_i, 2^-14) / w_i)).
    double part[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r)
        part[r] = (static_cast<double>(fabsf(X[r][0])) + fabsf(X[r][1])) + (static_cast<double>(fabsf(X[r][2])) + fabsf(X[r][3]));
    int slot;
    bool owner;
    const double rsum = row_reduce<Map<D>, double>(sm.rowbuf[warp], lane, part, slot, OpAdd());
    const int i_red = reduced_row<Map<D>>(warp, lane, slot, owner);
    if (owner) {
        const int bw = sm.bits[i_red];
        double m = rsum / D;
        if (m < kHalfMinNormal) m = kHalfMinNormal;
        double rr = m / static_cast<double>(sm.w[i_red]);
        rr = rr < kHalfMinNormal ? kHalfMinNormal : (rr > kHalfMax ? kHalfMax : rr);
        const __half rh = __double2half(rr);
        if (r_out) r_out[i_red] = __half_as_ushort(rh);
        const float rf = __half2float(rh);
        if (bw == 16) {
            // FP16 pivot row: no part in the shared column fit (a = 0 leaves the column max
            // alone, weight 0 leaves the least-squares sums alone).
            sm.rowa[i_red] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            const float a = 1.0f / (rf * static_cast<float>((1 << (8 - bw)) * qmax_of(bw)));
            const float ir = 1.0f / (rf * znorm_of(bw));
            sm.rowa[i_red] = make_float4(a, ir, sm.w[i_red], rf * znorm_of(bw));
        }
    }
    __syncwarp();

    // Column initialisation: c0_j = max(max_i |X_ij| a_i, 2^-14) (no entry clips).
    float cm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float a = sm.rowa[M::row(warp, lane, r)].x;
#pragma unroll
        for (int k = 0; k < 4; ++k) cm[k] = fmaxf(cm[k], __fmul_rn(fabsf(X[r][k]), a));
    }
    combine_subrows<Map<D>, float>(cm, OpMax());
    float* redf = reinterpret_cast<float*>(&sm.red[0][0][0]);
    if (lane < M::LPR)
#pragma unroll
        for (int k = 0; k < 4; ++k) redf[warp * D + 4 * cl + k] = cm[k];
    __syncthreads();
    if (tid < D) {
        float mx = 0.f;
#pragma unroll
        for (int w = 0; w < M::kWarps; ++w) mx = fmaxf(mx, redf[w * D + tid]);
        const float c0 = mx < kHalfMinNormal ? kHalfMinNormal : mx;
        sm.col0[tid] = c0;
        sm.colf[tid] = 1.0f / c0;
    }
    __syncthreads();

    // Codes at (r, c0) by the quantisation contract; one fixed-code weighted least-squares
    // update c_j = sum_i w_i^2 v_ij X_ij / sum_i w_i^2 v_ij^2, v_ij = r_i 2^(8-b_i) z0_ij.
    double num[4] = {0, 0, 0, 0}, den[4] = {0, 0, 0, 0};
    float ic0[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) ic0[k] = sm.colf[4 * cl + k];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = M::row(warp, lane, r);
        const float4 ra = sm.rowa[i];
        const int qb = qmax_of(sm.bits[i]);
        const double ww = static_cast<double>(ra.z) * static_cast<double>(ra.z);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int z0 = quantise(X[r][k], ra.y, ic0[k], qb);
            const double v = static_cast<double>(ra.w) * z0;
            num[k] += ww * v * static_cast<double>(X[r][k]);
            den[k] += ww * v * v;
        }
    }
    combine_subrows<Map<D>, double>(num, OpAdd());
    combine_subrows<Map<D>, double>(den, OpAdd());
    if (lane < M::LPR)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            sm.red[warp][0][4 * cl + k] = num[k];
            sm.red[warp][1][4 * cl + k] = den[k];
        }
    __syncthreads();
    if (tid < D) {
        double ns = 0, ds = 0;
#pragma unroll
        for (int w = 0; w < M::kWarps; ++w) {
            ns += sm.red[w][0][tid];
            ds += sm.red[w][1][tid];
        }
        double c1 = ds > 0 ? ns / ds : static_cast<double>(sm.col0[tid]);
        c1 = c1 < kHalfMinNormal ? kHalfMinNormal : (c1 > kHalfMax ? kHalfMax : c1);
        const __half ch = __double2half(c1);
        if (c_out) c_out[tid] = __half_as_ushort(ch);
        sm.colc[tid] = __half2float(ch);
        sm.colf[tid] = 1.0f / __half2float(ch);
    }
    __syncthreads();
}

struct StateArgs {
    int H;
    const float* S;
    const float* w;
    const uint8_t* bits;
    const int64_t* head_off;
    int64_t bytes_per_seq;
    uint16_t* r;
    uint16_t* c;
    const uint16_t* r_in;
    const uint16_t* c_in;
    uint8_t* packed;
    const uint8_t* packed_in;
    float* S_out;
    int uniform_bits;   // distortion: > 0 replaces the bit map by this width
    double* scratch;    // distortion: per-(tile, row) squared error
    uint32_t* flags;    // pack / unpack: device error word (bit 2: head range cannot hold the tile)
};

template <int D>
__device__ __forceinline__ void load_head(TileSmem<D>& sm, const StateArgs& a, int h) {
    const int tid = threadIdx.x;
    if (tid < D) {
        sm.bits[tid] = a.uniform_bits > 0 ? static_cast<uint8_t>(a.uniform_bits) : a.bits[h * D + tid];
        sm.w[tid] = a.w ? a.w[h * D + tid] : 1.0f;
    }
}

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads) fit_kernel(const StateArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(smem_raw);
    const int tile = blockIdx.x, h = tile % a.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    load_head<D>(sm, a, h);
    float X[M::RPT][4];
    load_tile<D>(a.S + static_cast<int64_t>(tile) * D * D, warp, lane, X);
    __syncthreads();
    fit_tile_regs<D>(sm, X, warp, lane, a.r + static_cast<int64_t>(tile) * D, a.c + static_cast<int64_t>(tile) * D);
}

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads) pack_kernel(const StateArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(smem_raw);
    const int tile = blockIdx.x, h = tile % a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    load_head<D>(sm, a, h);
    if (tid < D) {
        const int bw = a.bits[h * D + tid];
        const float rf = half_bits_to_float(a.r_in[static_cast<int64_t>(tile) * D + tid]);
        sm.rowa[tid] = make_float4(0.f, bw == 16 ? 0.f : 1.0f / (rf * znorm_of(bw)), 0.f, 0.f);
        sm.colf[tid] = 1.0f / half_bits_to_float(a.c_in[static_cast<int64_t>(tile) * D + tid]);
    }
    float X[M::RPT][4];
    load_tile<D>(a.S + static_cast<int64_t>(tile) * D * D, warp, lane, X);
    __syncthreads();
    if (warp == 0) {
        const int total = row_offsets_warp<D>(sm.bits, sm.roff, lane);
        if (lane == 0) sm.ok = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, total, 2 * D * D, a.flags);
    }
    __syncthreads();
    if (!sm.ok) return;   // offsets that do not match the bit map: nothing of the tile is written
    uint8_t* out = a.packed + static_cast<int64_t>(tile / a.H) * a.bytes_per_seq + a.head_off[h];
    float ic[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) ic[k] = sm.colf[4 * cl + k];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int i = M::row(warp, lane, r);
        const int bw = sm.bits[i];
        if (bw == 16) {   // FP16 pivot row
            __half2 h01 = __halves2half2(pivot_half(X[r][0]), pivot_half(X[r][1]));
            __half2 h23 = __halves2half2(pivot_half(X[r][2]), pivot_half(X[r][3]));
            *reinterpret_cast<uint2*>(out + sm.roff[i] + 8 * cl) =
                make_uint2(*reinterpret_cast<uint32_t*>(&h01), *reinterpret_cast<uint32_t*>(&h23));
            continue;
        }
        const float ir = sm.rowa[i].y;
        int q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = quantise(X[r][k], ir, ic[k], qmax_of(bw));
        pack4_store<D>(out + sm.roff[i], cl, bw, q);
    }
}

template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads) unpack_kernel(const StateArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(smem_raw);
    const int tile = blockIdx.x, h = tile % a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    load_head<D>(sm, a, h);
    if (tid < D) {
        sm.rowa[tid].x = half_bits_to_float(a.r_in[static_cast<int64_t>(tile) * D + tid]);
        sm.colc[tid] = half_bits_to_float(a.c_in[static_cast<int64_t>(tile) * D + tid]);
    }
    __syncthreads();
    if (warp == 0) {
        const int total = row_offsets_warp<D>(sm.bits, sm.roff, lane);
        if (lane == 0) sm.ok = tile_range_ok(a.head_off, a.H, a.bytes_per_seq, h, total, 2 * D * D, a.flags);
    }
    __syncthreads();
    if (!sm.ok) return;   // offsets that do not match the bit map: nothing of the tile is read
    const uint8_t* in = a.packed_in + static_cast<int64_t>(tile / a.H) * a.bytes_per_seq + a.head_off[h];
    float* S = a.S_out + static_cast<int64_t>(tile) * D * D;
    float cf[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) cf[k] = sm.colc[4 * cl + k];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int i = M::row(warp, lane, r);
        const int bw = sm.bits[i];
        const float rf = sm.rowa[i].x;
        float z[4];
        unpack4<D>(in + sm.roff[i], cl, bw, z);
        float x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            x[k] = bw == 16 ? z[k] : __fmul_rn(__fmul_rn(rf, cf[k]), __fmul_rn(z[k], znorm_of(bw)));
        *reinterpret_cast<float4*>(S + i * D + 4 * cl) = make_float4(x[0], x[1], x[2], x[3]);
    }
}

// Squared reconstruction error per row of each tile at a uniform width (fit, quantise,
// dequantise in registers).
template <int D>
__global__ void __launch_bounds__(Map<D>::kThreads) distortion_kernel(const StateArgs a) {
    using M = Map<D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(smem_raw);
    const int tile = blockIdx.x, h = tile % a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cl = M::col_lane(lane);
    load_head<D>(sm, a, h);
    float X[M::RPT][4];
    load_tile<D>(a.S + static_cast<int64_t>(tile) * D * D, warp, lane, X);
    __syncthreads();
    fit_tile_regs<D>(sm, X, warp, lane, nullptr, nullptr);
    double part[M::RPT];
#pragma unroll
    for (int r = 0; r < M::RPT; ++r) {
        const int i = M::row(warp, lane, r);
        const int bw = sm.bits[i];
        const float4 ra = sm.rowa[i];
        double acc = 0;
        if (bw == 16) {   // FP16 pivot row: the binary16 rounding error
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const double e = static_cast<double>(__half2float(pivot_half(X[r][k]))) - static_cast<double>(X[r][k]);
                acc += e * e;
            }
        } else {
            const int qb = qmax_of(bw);
            const float zn = znorm_of(bw);
            const float rf = ra.w / zn;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int q = quantise(X[r][k], ra.y, sm.colf[4 * cl + k], qb);
                const float xh = __fmul_rn(__fmul_rn(rf, sm.colc[4 * cl + k]), static_cast<float>(q) * zn);
                const double e = static_cast<double>(xh) - static_cast<double>(X[r][k]);
                acc += e * e;
            }
        }
        part[r] = acc;
    }
    int slot;
    bool owner;
    const double rs = row_reduce<Map<D>, double>(sm.rowbuf[warp], lane, part, slot, OpAdd());
    const int i = reduced_row<Map<D>>(warp, lane, slot, owner);
    if (owner) a.scratch[static_cast<int64_t>(tile) * D + i] = rs;
}

// d_row[h][i] = sum_b scratch[b][h][i] / (B D); d_head[h] = sum_i w_i^2 (...) / (B D D).
template <int D>
__global__ void distortion_finish_kernel(int B, int H, const double* scratch, const float* w, double* d_row,
                                         double* d_head) {
    __shared__ double part[D];
    const int h = blockIdx.x, i = threadIdx.x;
    double acc = 0;
    for (int b = 0; b < B; ++b) acc += scratch[(static_cast<int64_t>(b) * H + h) * D + i];
    d_row[h * D + i] = acc / (static_cast<double>(B) * D);
    const double wi = w[h * D + i];
    part[i] = wi * wi * acc;
    __syncthreads();
    if (i == 0) {
        double s = 0;
        for (int k = 0; k < D; ++k) s += part[k];
        d_head[h] = s / (static_cast<double>(B) * D * D);
    }
}

template <int D>
static int launch_state(const char* fn, void (*kern)(StateArgs), int tiles, const StateArgs& a, cudaStream_t st) {
    if (tiles == 0) return STEPQ_OK;
    const size_t smem = sizeof(TileSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
    kern<<<tiles, Map<D>::kThreads, smem, st>>>(a);
    return check_launch(fn);
}

static int common_checks(const stepq_dims& d, const char* fn, long long& tiles) {
    int rc = check_dims(d, fn);
    if (rc) return rc;
    tiles = static_cast<long long>(d.B) * d.H;
    if (tiles > 0x7fffffffLL) return set_error(STEPQ_EINVAL, "%s: too many tiles", fn);
    return STEPQ_OK;
}

}  // namespace stepq

using namespace stepq;

extern "C" int stepq_fit_scales(stepq_dims dims, const float* S, const float* w, const uint8_t* bits, uint16_t* r,
                                uint16_t* c, void* stream) {
    clear_error();
    long long tiles;
    int rc = common_checks(dims, "stepq_fit_scales", tiles);
    if (rc || tiles == 0) return rc;
    rc = check_ptrs("stepq_fit_scales", {{"S", S}, {"w", w}, {"bits", bits}, {"r", r}, {"c", c}});
    if (rc) return rc;
    StateArgs a{};
    a.H = dims.H; a.S = S; a.w = w; a.bits = bits; a.r = r; a.c = c;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128 ? launch_state<128>("stepq_fit_scales", fit_kernel<128>, (int)tiles, a, st)
                          : launch_state<64>("stepq_fit_scales", fit_kernel<64>, (int)tiles, a, st);
}

extern "C" int stepq_pack_state(stepq_dims dims, const float* S, const uint8_t* bits, const int64_t* head_off,
                                int64_t bytes_per_seq, const uint16_t* r, const uint16_t* c, uint8_t* packed,
                                void* stream) {
    clear_error();
    long long tiles;
    int rc = common_checks(dims, "stepq_pack_state", tiles);
    if (rc || tiles == 0) return rc;
    rc = check_ptrs("stepq_pack_state",
                    {{"S", S}, {"bits", bits}, {"head_off", head_off}, {"r", r}, {"c", c}, {"packed", packed}});
    if (rc) return rc;
    if (bytes_per_seq <= 0 || (bytes_per_seq & 15))
        return set_error(STEPQ_EINVAL, "stepq_pack_state: bytes_per_seq=%lld", (long long)bytes_per_seq);
    StateArgs a{};
    a.H = dims.H; a.S = S; a.bits = bits; a.head_off = head_off; a.bytes_per_seq = bytes_per_seq;
    a.r_in = r; a.c_in = c; a.packed = packed;
    rc = device_flags_ptr(&a.flags);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128 ? launch_state<128>("stepq_pack_state", pack_kernel<128>, (int)tiles, a, st)
                          : launch_state<64>("stepq_pack_state", pack_kernel<64>, (int)tiles, a, st);
}

extern "C" int stepq_unpack_state(stepq_dims dims, const uint8_t* packed, const uint8_t* bits,
                                  const int64_t* head_off, int64_t bytes_per_seq, const uint16_t* r,
                                  const uint16_t* c, float* S_out, void* stream) {
    clear_error();
    long long tiles;
    int rc = common_checks(dims, "stepq_unpack_state", tiles);
    if (rc || tiles == 0) return rc;
    rc = check_ptrs("stepq_unpack_state",
                    {{"packed", packed}, {"bits", bits}, {"head_off", head_off}, {"r", r}, {"c", c}, {"S_out", S_out}});
    if (rc) return rc;
    if (bytes_per_seq <= 0 || (bytes_per_seq & 15))
        return set_error(STEPQ_EINVAL, "stepq_unpack_state: bytes_per_seq=%lld", (long long)bytes_per_seq);
    StateArgs a{};
    a.H = dims.H; a.bits = bits; a.head_off = head_off; a.bytes_per_seq = bytes_per_seq;
    a.r_in = r; a.c_in = c; a.packed_in = packed; a.S_out = S_out;
    rc = device_flags_ptr(&a.flags);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims.dk == 128 ? launch_state<128>("stepq_unpack_state", unpack_kernel<128>, (int)tiles, a, st)
                          : launch_state<64>("stepq_unpack_state", unpack_kernel<64>, (int)tiles, a, st);
}

extern "C" int stepq_calib_distortion(stepq_dims dims, const float* S, const float* w, int b, double* d_row,
                                      double* d_head, double* scratch, void* stream) {
    clear_error();
    long long tiles;
    int rc = common_checks(dims, "stepq_calib_distortion", tiles);
    if (rc) return rc;
    if (b != 2 && b != 4 && b != 6 && b != 8 && b != 16)
        return set_error(STEPQ_EUNSUPPORTED, "stepq_calib_distortion: width %d", b);
    if (tiles == 0) return set_error(STEPQ_EINVAL, "stepq_calib_distortion: no sample states (B=0)");
    rc = check_ptrs("stepq_calib_distortion",
                    {{"S", S}, {"w", w}, {"d_row", d_row}, {"d_head", d_head}, {"scratch", scratch}});
    if (rc) return rc;
    StateArgs a{};
    a.H = dims.H; a.S = S; a.w = w; a.uniform_bits = b; a.scratch = scratch;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.dk == 128) {
        rc = launch_state<128>("stepq_calib_distortion", distortion_kernel<128>, (int)tiles, a, st);
        if (rc) return rc;
        distortion_finish_kernel<128><<<dims.H, 128, 0, st>>>(dims.B, dims.H, scratch, w, d_row, d_head);
    } else {
        rc = launch_state<64>("stepq_calib_distortion", distortion_kernel<64>, (int)tiles, a, st);
        if (rc) return rc;
        distortion_finish_kernel<64><<<dims.H, 64, 0, st>>>(dims.B, dims.H, scratch, w, d_row, d_head);
    }
    return check_launch("stepq_calib_distortion");
}

extern "C" int stepq_calib_distortion_bits(stepq_dims dims, const float* S, const float* w, const uint8_t* bits,
                                           double* d_row, double* d_head, double* scratch, void* stream) {
    const char* fn = "stepq_calib_distortion_bits";
    clear_error();
    long long tiles;
    int rc = common_checks(dims, fn, tiles);
    if (rc) return rc;
    if (tiles == 0) return set_error(STEPQ_EINVAL, "%s: no sample states (B=0)", fn);
    rc = check_ptrs(fn, {{"S", S}, {"w", w}, {"bits", bits}, {"d_row", d_row}, {"d_head", d_head}, {"scratch", scratch}});
    if (rc) return rc;
    StateArgs a{};
    a.H = dims.H; a.S = S; a.w = w; a.bits = bits; a.uniform_bits = 0; a.scratch = scratch;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.dk == 128) {
        rc = launch_state<128>(fn, distortion_kernel<128>, (int)tiles, a, st);
        if (rc) return rc;
        distortion_finish_kernel<128><<<dims.H, 128, 0, st>>>(dims.B, dims.H, scratch, w, d_row, d_head);
    } else {
        rc = launch_state<64>(fn, distortion_kernel<64>, (int)tiles, a, st);
        if (rc) return rc;
        distortion_finish_kernel<64><<<dims.H, 64, 0, st>>>(dims.B, dims.H, scratch, w, d_row, d_head);
    }
    return check_launch(fn);
}

namespace stepq {

// Work space of stepq_calib_distortion_static: the squared error of each (sample state, head,
// key row), written by the distortion kernel and summed by its finishing kernel. Host code
// reaches it only through the address cudaGetSymbolAddress returns.
static __device__ __align__(256) double g_distortion_scratch[STEPQ_STATIC_SCRATCH_ROWS];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mutex;
static double* g_scratch_addr[kMaxDevices];

// The current device's copy of the work space, looked up on the first call for that device.
static int static_scratch(const char* fn, double** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: cudaGetDevice: %s", fn, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return set_error(STEPQ_EUNSUPPORTED, "%s: device ordinal %d", fn, dev);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_distortion_scratch);
        if (e != cudaSuccess || p == nullptr)
            return set_error(STEPQ_ECUDA, "%s: cudaGetSymbolAddress: %s", fn, cudaGetErrorString(e));
        g_scratch_addr[dev] = static_cast<double*>(p);
    }
    *out = g_scratch_addr[dev];
    return STEPQ_OK;
}

}  // namespace stepq

extern "C" int stepq_calib_distortion_static(stepq_dims dims, const float* S, const float* w, int b, double* d_row,
                                             double* d_head, void* stream) {
    const char* fn = "stepq_calib_distortion_static";
    clear_error();
    long long tiles;
    int rc = common_checks(dims, fn, tiles);
    if (rc) return rc;
    if (b != 2 && b != 4 && b != 6 && b != 8 && b != 16) return set_error(STEPQ_EUNSUPPORTED, "%s: width %d", fn, b);
    if (tiles == 0) return set_error(STEPQ_EINVAL, "%s: no sample states (B=0)", fn);
    if (tiles * dims.dk > STEPQ_STATIC_SCRATCH_ROWS)
        return set_error(STEPQ_EINVAL, "%s: B*H*dk = %lld exceeds the static work space of %d entries", fn,
                         tiles * dims.dk, STEPQ_STATIC_SCRATCH_ROWS);
    rc = check_ptrs(fn, {{"S", S}, {"w", w}, {"d_row", d_row}, {"d_head", d_head}});
    if (rc) return rc;
    double* scratch = nullptr;
    rc = static_scratch(fn, &scratch);
    if (rc) return rc;
    StateArgs a{};
    a.H = dims.H; a.S = S; a.w = w; a.uniform_bits = b; a.scratch = scratch;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.dk == 128) {
        rc = launch_state<128>(fn, distortion_kernel<128>, (int)tiles, a, st);
        if (rc) return rc;
        distortion_finish_kernel<128><<<dims.H, 128, 0, st>>>(dims.B, dims.H, scratch, w, d_row, d_head);
    } else {
        rc = launch_state<64>(fn, distortion_kernel<64>, (int)tiles, a, st);
        if (rc) return rc;
        distortion_finish_kernel<64><<<dims.H, 64, 0, st>>>(dims.B, dims.H, scratch, w, d_row, d_head);
    }
    return check_launch(fn);
}
