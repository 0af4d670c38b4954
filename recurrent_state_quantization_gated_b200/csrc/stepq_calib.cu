// stepq_calib.cu -- offline row-impact calibration of STEPQuant (App. B.3, App. C.1) on sm_100a.
//
// omega_{h,i} = E over the calibration stream of (A_t^T q_t)_i^2, where
// (A_t^T q_t)_i = d_{t,i} (q_{t,i} - beta_t k_{t,i} (k_t . q_t)) is the immediate Delta
// transition followed by the readout. The key-row impact factor is w_i = omega_i^(1/8),
// normalised to mean 1 within each head, with a numerical floor of 1e-12 max_i omega_i.
//
// One CTA per head; each warp walks a fixed, strided subset of the (step, sequence) samples and
// accumulates in float64, so the result is deterministic.
#include <cuda_runtime.h>

#include "stepq_device.cuh"
#include "stepq_internal.h"

namespace stepq {

template <int D>
__global__ void __launch_bounds__(256) row_impact_kernel(int T, int B, int H, int gpc, const uint16_t* q,
                                                         const uint16_t* k, const float* beta, const float* gate,
                                                         float* w_out) {
    constexpr int RL = D / 32;
    constexpr int NW = 8;
    __shared__ double acc_s[NW][D];
    __shared__ double red[NW];
    const int h = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double acc[RL];
#pragma unroll
    for (int r = 0; r < RL; ++r) acc[r] = 0;
    const long long samples = static_cast<long long>(T) * B;
    for (long long s = warp; s < samples; s += NW) {
        const long long tile = s * H + h;
        double qv[RL], kv[RL], kq = 0;
#pragma unroll
        for (int r = 0; r < RL; ++r) {
            const int i = lane * RL + r;
            qv[r] = bf16_bits_to_float(q[tile * D + i]);
            kv[r] = bf16_bits_to_float(k[tile * D + i]);
            kq += kv[r] * qv[r];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
        const double bt = beta[tile];
#pragma unroll
        for (int r = 0; r < RL; ++r) {
            const int i = lane * RL + r;
            const double d = gpc ? gate[tile * D + i] : gate[tile];
            const double g = d * (qv[r] - bt * kv[r] * kq);
            acc[r] += g * g;
        }
    }
#pragma unroll
    for (int r = 0; r < RL; ++r) acc_s[warp][lane * RL + r] = acc[r];
    __syncthreads();
    const int i = threadIdx.x;
    double om = 0;
    if (i < D) {
        for (int w = 0; w < NW; ++w) om += acc_s[w][i];
        om /= static_cast<double>(samples);
    }
    // max over the head's rows
    double mx = (i < D) ? om : 0;
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = 0;
    for (int w = 0; w < NW; ++w) mx = fmax(mx, red[w]);
    __syncthreads();
    double wv = 0;
    if (i < D) {
        if (om < 1e-12 * mx) om = 1e-12 * mx;
        wv = pow(om, 0.125);
    }
    double sm = wv;
    for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
    if (lane == 0) red[warp] = sm;
    __syncthreads();
    double mean = 0;
    for (int w = 0; w < NW; ++w) mean += red[w];
    mean /= D;
    if (i < D) w_out[h * D + i] = static_cast<float>(mean > 0 ? wv / mean : 1.0);
}

}  // namespace stepq

using namespace stepq;

extern "C" int stepq_row_impact(stepq_dims dims, int T, const uint16_t* q, const uint16_t* k, const float* beta,
                                const float* gate, float* w_out, void* stream) {
    clear_error();
    int rc = check_dims(dims, "stepq_row_impact");
    if (rc) return rc;
    if (T <= 0 || dims.B <= 0) return set_error(STEPQ_EINVAL, "stepq_row_impact: T=%d B=%d", T, dims.B);
    rc = check_ptrs("stepq_row_impact", {{"q", q}, {"k", k}, {"beta", beta}, {"gate", gate}, {"w_out", w_out}});
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dims.dk == 128)
        row_impact_kernel<128><<<dims.H, 256, 0, st>>>(T, dims.B, dims.H, dims.gate_per_channel, q, k, beta, gate, w_out);
    else
        row_impact_kernel<64><<<dims.H, 256, 0, st>>>(T, dims.B, dims.H, dims.gate_per_channel, q, k, beta, gate, w_out);
    return check_launch("stepq_row_impact");
}
