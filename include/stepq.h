/*
 * stepq.h -- C ABI of libstepq: STEPQuant's quantized gated Delta-rule decode step on B200.
 *
 * The method is the one of "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
 * State Quantization": a per-(sequence, head) recurrent state S (d_k x d_v, row = key
 * channel, column = value channel) kept as mixed-precision integer codes with a bit width per
 * key row and binary16 row and column scales, updated once per decoded token by the gated
 * Delta rule (§2.1) and re-quantised in place (App. C.3, Table C2).
 *
 * Conventions for every call below.
 *   - Pointers are DEVICE pointers unless the name ends in _host. They are owned by the caller
 *     and must stay valid until the work queued on `stream` has finished. The library never
 *     allocates or frees memory and never synchronises; every device call is queued on
 *     `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - Device pointers must be 16-byte aligned (STEPQ_EALIGN otherwise); packed buffers must
 *     also have a 16-byte aligned base.
 *   - d_k = d_v = 64 or 128 (STEPQ_EUNSUPPORTED otherwise); bit widths are 2, 4, 6 or 8, or
 *     16 for an FP16 pivot row (App. C.2; Table C2 steps 1 and 6), which keeps its values in
 *     binary16 and takes no part in the shared column fit.
 *   - Arrays are row-major: S float32 [B][H][dk][dv]; q, k bf16 bits (uint16) [B][H][dk];
 *     v bf16 bits [B][H][dv]; beta float32 [B][H]; gate float32 [B][H] (scalar gate per head,
 *     GDN) or [B][H][dk] (one gate per key channel, KDA; dims.gate_per_channel = 1);
 *     bits uint8 [H][dk]; w float32 [H][dk]; r binary16 bits [B][H][dk]; c binary16 bits
 *     [B][H][dv]; o float32 [B][H][dv].
 *   - Packed state: tile (b, h) starts at byte b * bytes_per_seq + head_off[h]; a row of
 *     width b takes dv*b/8 bytes; the integer rows come first, in key order, then the FP16
 *     pivot rows, in key order. Codes are b-bit two's complement integers q in [-q_b, q_b],
 *     q_b = 2^(b-1)-1. A 2- or 8-bit row stores column j at bit j*b of a little-endian bit
 *     stream; a 4-bit row stores columns 4g..4g+3 in the little-endian halfword g, column
 *     4g+m at bit 4*pos(m), pos = (0, 2, 1, 3); a 6-bit row stores the low 4 bits of every
 *     code (laid out as a 4-bit row) followed by the high 2 bits (laid out as a 2-bit row).
 *     A pivot row stores column j as binary16 at byte 2j.
 *   - Reconstruction (dequantisation), fp32: x_hat_ij = (r_i * c_j) * (q_ij * 2^(8-b_i)),
 *     i.e. the code normalisation z = 2^(8-b) q of App. C.1 with scales X_hat = r_i c_j z_ij
 *     (§4.3).
 *   - Quantisation, fp32: t = (x * ir_i) * ic_j with ir_i = 1/(r_i 2^(8-b_i)), ic_j = 1/c_j;
 *     q = clamp(rint(t), -q_b, q_b), rint rounding to nearest, ties to even (§2.2). A pivot
 *     entry is x rounded to binary16 (nearest-even, saturating at +-65504); its row factor is
 *     computed like any other and not used.
 *   - Return value: STEPQ_OK or an error code; stepq_last_error() then describes it (per
 *     thread). On an error nothing has been queued.
 */
#ifndef STEPQ_H
#define STEPQ_H

#include <stdint.h>

#if defined(__GNUC__)
#define STEPQ_API __attribute__((visibility("default")))
#else
#define STEPQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    STEPQ_OK = 0,
    STEPQ_EINVAL = 1,        /* bad argument (null pointer, negative size, ...)            */
    STEPQ_EUNSUPPORTED = 2,  /* d_k / d_v not in {64, 128}, or a width not in {2,4,6,8,16} */
    STEPQ_EALIGN = 3,        /* a device pointer is not 16-byte aligned                     */
    STEPQ_EBUDGET = 4,       /* bit allocation: no assignment reaches the budget exactly    */
    STEPQ_ECUDA = 5          /* a CUDA launch failed; stepq_last_error() names the error    */
};

typedef struct {
    int B;                   /* sequences                                    */
    int H;                   /* heads                                        */
    int dk;                  /* key width (rows of a state tile)             */
    int dv;                  /* value width (columns of a state tile)        */
    int gate_per_channel;    /* 0: gate [B][H]; 1: gate [B][H][dk]           */
    int pivots;              /* 1: the bit map may hold width-16 (FP16 pivot) rows. Read by the
                                decode steps and the prefill chunks, which then run their
                                pivot-capable kernels; a pivot row met with pivots = 0 raises
                                bit 1 of the device error word and its results are undefined.
                                Other calls ignore it.  */
    int mixed;               /* 1: some head's key rows have different widths (a row-level bit
                                allocation). Read by stepq_decode_step and the sequential prefill
                                chunk, which then run one code path for every row width instead of width-specialised paths per
                                warp (smaller code: faster for such maps, slower for maps whose
                                heads each use one width). Results are identical either way.  */
    int widths;              /* The row widths the bit map holds, as a bit mask (bit b set for
                                width b: 2, 4, 6, 8, 16), or 0 when not declared. Read by
                                stepq_decode_step with mixed = 1, whose per-row code then handles
                                only the declared widths (less code: the {2, 4, 8} and {4, 6, 8}
                                sets have their own kernels). A row of an undeclared width is
                                decoded as one of the declared ones and its results are undefined;
                                every access stays inside its tile. Other bits: STEPQ_EINVAL.
                                Other calls ignore it.  */
} stepq_dims;

/* Text of the last error raised on the calling thread ("" if none). */
STEPQ_API const char* stepq_last_error(void);

/* Host only. Packed layout of a bit map (the per-key-row widths of §3.2, frozen offline and
   shared by all sequences, App. C.2): head_off_host[h] = byte offset of head h inside one
   sequence, *bytes_per_seq, *total_bytes = B * bytes_per_seq. Any of the three outputs may
   be NULL. Scale storage (fp16 r and c, App. D Eq. 22) is separate and not counted. */
STEPQ_API int stepq_packed_layout(stepq_dims dims, const uint8_t* bits_host, int64_t* head_off_host,
                        int64_t* bytes_per_seq, int64_t* total_bytes);

/* Key-row-aware dual-axis fit (§4.3 "Row factors" / "Column factors", App. C.1) of every
   state tile: r_i = fp16(clamp(max(mean_j |S_ij|, 2^-14) / w_i, 2^-14, 65504)); the column
   scales start at the smallest value at which no entry clips, c0_j = max(max_i |S_ij| /
   (r_i 2^(8-b_i) q_b), 2^-14); codes z0 at (r, c0); then one fixed-code weighted
   least-squares update c_j = sum_i w_i^2 v_ij S_ij / sum_i w_i^2 v_ij^2 (v_ij = r_i 2^(8-b_i)
   z0_ij; a zero denominator keeps c0_j), rounded to fp16 after clamping into [2^-14, 65504].
   Outputs r [B][H][dk], c [B][H][dv]. */
STEPQ_API int stepq_fit_scales(stepq_dims dims, const float* S, const float* w, const uint8_t* bits,
                     uint16_t* r, uint16_t* c, void* stream);

/* Quantise S with the given scales and write the packed codes (the quantisation contract
   above; §2.2 and §4.3 "Quantization"). head_off is the device copy of stepq_packed_layout's
   head offsets. */
STEPQ_API int stepq_pack_state(stepq_dims dims, const float* S, const uint8_t* bits, const int64_t* head_off,
                     int64_t bytes_per_seq, const uint16_t* r, const uint16_t* c, uint8_t* packed,
                     void* stream);

/* Reconstruct S_out (float32 [B][H][dk][dv]) from packed codes and scales (dequantisation
   contract above; §4.3, App. C.1). */
STEPQ_API int stepq_unpack_state(stepq_dims dims, const uint8_t* packed, const uint8_t* bits,
                       const int64_t* head_off, int64_t bytes_per_seq, const uint16_t* r,
                       const uint16_t* c, float* S_out, void* stream);

/* One persistent decode step of every tile (Table C2), fused in one kernel that reads the
   packed state from HBM once and writes it once:
     1. reconstruct S_hat from packed_in, r_in, c_in;
     2. X = D S_hat + beta k (v^T - k^T D S_hat)   (gated Delta rule, §2.1; D = gate);
     3. o = X^T q, before requantisation (Table C2 step 3);
     4.-5. refit r, c on X exactly as stepq_fit_scales (key-row impact w, §4.3, App. C.1);
     6. quantise X with the new scales and write packed_out, r_out, c_out.
   packed_out may equal packed_in, r_out may equal r_in and c_out may equal c_in (in-place
   update: each tile is read completely before any of it is written). Arithmetic is fp32; the
   result matches a float64 evaluation of steps 1-3 to ~1e-6 relative, and the requantised
   codes may differ from that evaluation's by one step where an entry lies on a rounding
   boundary. */
STEPQ_API int stepq_decode_step(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const float* beta, const float* gate, const uint8_t* bits, const float* w,
                      const int64_t* head_off, int64_t bytes_per_seq, const uint8_t* packed_in,
                      const uint16_t* r_in, const uint16_t* c_in, uint8_t* packed_out,
                      uint16_t* r_out, uint16_t* c_out, float* o, void* stream);

/* A prefill chunk on the packed state (STEPQuant App. F.1 "prefill unpacks active states,
   runs the native chunk kernel, and packs the resulting boundary states"; App. B.2): per tile,
   reconstruct S_hat once, apply the gated Delta rule for `chunk` tokens in fp32 without
   requantising in between (readout o_t = X_t^T q_t after each token), then refit and pack the
   boundary state once, as steps 4-6 of stepq_decode_step. Token inputs and o carry a leading
   token axis: q, k [chunk][B][H][dk], v [chunk][B][H][dv], beta [chunk][B][H], gate
   [chunk][B][H] or [chunk][B][H][dk], o [chunk][B][H][dv]. In-place use and dims.pivots as for
   stepq_decode_step.
   Two forms compute it:
     stepq_prefill_chunk_seq: the tokens one after another on the register-resident tile (any
       supported shape and chunk length; chunk = 1 is bit-identical to stepq_decode_step);
     stepq_prefill_chunk_wy: the chunked WY/UT form on the tensor cores (§2.1's affine form
       unrolled over the chunk: one unit lower triangular solve and dense products per tile).
       Requires dk = dv = 128 and 1 <= chunk <= STEPQ_WY_MAX_CHUNK; otherwise
       STEPQ_EUNSUPPORTED. Scalar and channel gates (gates in [0, 1]); FP16 pivot rows enter the
       products as v_ij / c_j in two bf16 parts and the boundary state from their stored values. Products run on
       bf16 operands (q, k, v and the integer codes exactly; computed operands split into two or
       three bf16 parts) with fp32 accumulation; under channel gates the gate-weighted token-pair
       products (the triangular system's and the readouts' intra-chunk weights) are formed on
       the CUDA cores in fp32. The boundary
       state carries fp32 precision, the readouts about 1e-6 relative.
   stepq_prefill_chunk takes the WY form for dk = dv = 128, scalar gates and chunk <=
   STEPQ_WY_MAX_CHUNK (FP16 pivot rows or not), and the sequential form elsewhere: under channel
   gates the WY form's pair products on the CUDA cores make it the slower of the two. */
#define STEPQ_WY_MAX_CHUNK 64
STEPQ_API int stepq_prefill_chunk(stepq_dims dims, int chunk, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const float* beta, const float* gate, const uint8_t* bits,
                        const float* w, const int64_t* head_off, int64_t bytes_per_seq,
                        const uint8_t* packed_in, const uint16_t* r_in, const uint16_t* c_in,
                        uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out, float* o, void* stream);
STEPQ_API int stepq_prefill_chunk_seq(stepq_dims dims, int chunk, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const float* beta, const float* gate, const uint8_t* bits,
                        const float* w, const int64_t* head_off, int64_t bytes_per_seq,
                        const uint8_t* packed_in, const uint16_t* r_in, const uint16_t* c_in,
                        uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out, float* o, void* stream);
STEPQ_API int stepq_prefill_chunk_wy(stepq_dims dims, int chunk, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const float* beta, const float* gate, const uint8_t* bits,
                        const float* w, const int64_t* head_off, int64_t bytes_per_seq,
                        const uint8_t* packed_in, const uint16_t* r_in, const uint16_t* c_in,
                        uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out, float* o, void* stream);

/* The split form of the same step (STEPQuant §4.4 and App. F.1: reconstruction, the update and
   the readout fused; scale fitting and packed writeback run afterwards on a separate stream),
   kept as an ablation of the single fused kernel:
     on `stream`: one kernel does steps 1-3 of stepq_decode_step and writes o and the updated
       state X (float32 [B][H][dk][dv]) into the caller's work space x_ws (64 KiB per tile at
       d = 128);
     on `side_stream`, ordered after that kernel by an event the library records on `stream`:
       stepq_fit_scales(x_ws) -> r_out, c_out and stepq_pack_state(x_ws) -> packed_out.
   The results equal the fused step's within its stated tolerance (o identically). The side
   stream's work must complete before anything reads packed_out, r_out, c_out or reuses x_ws:
   the caller orders that (e.g. an event recorded on side_stream after this call). Passing
   packed_out, r_out and c_out all NULL runs the first kernel only (o and X). In-place use as
   for stepq_decode_step. The library keeps one event per device, created on the first call. */
STEPQ_API int stepq_decode_step_split(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const float* beta, const float* gate, const uint8_t* bits, const float* w,
                            const int64_t* head_off, int64_t bytes_per_seq, const uint8_t* packed_in,
                            const uint16_t* r_in, const uint16_t* c_in, uint8_t* packed_out,
                            uint16_t* r_out, uint16_t* c_out, float* o, float* x_ws, void* stream,
                            void* side_stream);

/* FP32-state decode step (the unquantised state of §5.1): S_out = D S + beta k (v^T - k^T D S),
   o = S_out^T q. S_out may equal S_in. */
STEPQ_API int stepq_decode_step_fp32(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const float* beta, const float* gate, const float* S_in, float* S_out,
                           float* o, void* stream);

/* Uniform symmetric rowwise-absmax INT8 state (the baseline of §5.1): codes int8
   [B][H][dk][dv], row scales s binary16 [B][H][dk], x_hat = s_i * q;
   s_i = fp16(clamp(max_j |X_ij| / 127, 2^-14, 65504)), q = clamp(rint(X * (1/s_i)), -127, 127).
   stepq_int8_quantize_state quantises S; stepq_decode_step_int8 is the decode step on that
   format (dequantise, gated Delta update, readout before requantisation, requantise).
   Outputs may alias the inputs. */
STEPQ_API int stepq_int8_quantize_state(stepq_dims dims, const float* S, int8_t* codes, uint16_t* s, void* stream);
STEPQ_API int stepq_decode_step_int8(stepq_dims dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const float* beta, const float* gate, const int8_t* codes_in,
                           const uint16_t* s_in, int8_t* codes_out, uint16_t* s_out, float* o,
                           void* stream);

/* One token of the per-window 8-bit state (LeapQuant's abstract on the page "When Dynamic Scaling
   Fails: A Scale-State Feedback Governs Recurrent-State Quantization in Linear-Attention and SSM
   LLMs": quantise the state once at the end of a window of tokens; inside the window the readouts
   come from the fixed low-bit state plus high-precision buffered updates). The state
   between windows is the rowwise-absmax INT8 format above (codes, s). Token t of the window
   (0 <= t < window <= STEPQ_LEAP_MAX_WINDOW) reads codes and s and the window's buffers entries
   0 .. t-1, and writes entry t:
     kbuf  bf16 [window][B][H][dk]  the window's keys,
     ubuf  fp32 [window][B][H][dv]  the pseudo-values u_r = beta_r (v_r - g_r S_{r-1}^T k_r),
     lbuf  fp32 [window][B][H]      the running log2 of the gate product (a zero gate counts 2^-64).
   With gamma_r = 2^lbuf_r: o_t = S_t^T q_t with S_t = gamma_t S_hat + sum_{r<=t} (gamma_t/gamma_r)
   k_r u_r^T, all in fp32; the last token (t = window - 1) also writes that state, requantised,
   over codes and s. Scalar gates only (dims.gate_per_channel = 1 is STEPQ_EUNSUPPORTED); the
   buffers belong to the caller and must not be changed while a window is open. */
#define STEPQ_LEAP_MAX_WINDOW 256
STEPQ_API int stepq_leap_step(stepq_dims dims, int window, int t, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, const float* beta, const float* gate, int8_t* codes, uint16_t* s,
                    uint16_t* kbuf, float* ubuf, float* lbuf, float* o, void* stream);

/* Offline calibration (not on the decode path).
   Row impact (App. B.3, C.1) over a calibration stream of T steps, arrays with a leading
   step axis ([T][B][H]...): omega_{h,i} = mean_{t,b} (d_{t,i} (q_{t,i} - beta_t k_{t,i}
   (k_t . q_t)))^2, floored at 1e-12 max_i omega_{h,i}; w_out[h][i] = omega^(1/8) normalised to
   mean 1 per head. dims.B is the number of sequences per step. */
STEPQ_API int stepq_row_impact(stepq_dims dims, int T, const uint16_t* q, const uint16_t* k,
                     const float* beta, const float* gate, float* w_out, void* stream);

/* Candidate-format distortion (App. A.3, Eq. 17 and Eq. 18) of the sample states S
   [B][H][dk][dv] quantised at the uniform width b with the fit of stepq_fit_scales:
   d_row[h][i] = (1/(B dv)) sum_{b,j} (x_hat - x)^2 and
   d_head[h] = (1/(B dk dv)) sum_{b,i,j} w_i^2 (x_hat - x)^2 (float64, device).
   scratch: caller-provided float64 [B][H][dk] work space. */
STEPQ_API int stepq_calib_distortion(stepq_dims dims, const float* S, const float* w, int b, double* d_row,
                           double* d_head, double* scratch, void* stream);

/* The same under a per-row bit map bits [H][dk] (widths 2, 4, 6, 8 and 16 = FP16 pivot rows,
   which take no part in the shared column fit): the candidate distortions recalibrated with
   the pivots fixed (App. C.2, KDA calibration). */
STEPQ_API int stepq_calib_distortion_bits(stepq_dims dims, const float* S, const float* w, const uint8_t* bits,
                                double* d_row, double* d_head, double* scratch, void* stream);

/* Capacity, in float64 entries, of the static work space of stepq_calib_distortion_static:
   it takes B * H * dk <= STEPQ_STATIC_SCRATCH_ROWS (4 MiB of device memory per device, held
   by the loaded library). */
#define STEPQ_STATIC_SCRATCH_ROWS 524288

/* stepq_calib_distortion without the caller's work space, allocating nothing. No counterpart
   in the paper: it exists for callers that may not allocate device memory when they measure
   distortion, such as a process whose device memory is already reserved in full (a serving
   process that sized its pool for the packed states and caches) or one that runs under an
   allocator which forbids new device allocations after start-up; they cannot hand over the
   [B][H][dk] work space of stepq_calib_distortion.
   The work space is a file-scope device array of STEPQ_STATIC_SCRATCH_ROWS float64 entries,
   one per device. The first call on each device (with that device current) looks up its
   address with cudaGetSymbolAddress; make that first call before any stream capture. The
   address is kept for the life of the process: after cudaDeviceReset() of a device (which
   unloads the library's device code there) this entry point must not be called on that device
   again in the same process. Every
   entry the call reads it has written itself, so nothing in the array needs clearing.
   All calls on one device share the array: calls that overlap in time (on different streams,
   or from different host threads without ordering) race and give wrong results; order them
   on one stream. Arguments, layout and results are those of stepq_calib_distortion.
   Returns STEPQ_EINVAL when B * H * dk exceeds STEPQ_STATIC_SCRATCH_ROWS (nothing is
   launched), STEPQ_ECUDA when the address lookup or a launch fails. */
STEPQ_API int stepq_calib_distortion_static(stepq_dims dims, const float* S, const float* w, int b,
                                  double* d_row, double* d_head, void* stream);

/* Host only. Lifetime-aware bit allocation (§3.2, App. C.2): widths bits_out_host[u] from the
   ascending candidates cand_host[0..n_cand) minimising sum_u J_host[u][k] with exactly
   budget_bits bits in total (J is the lifetime-weighted distortion L_u d_u(b)).
   mode 1: multiple-choice dynamic programme (the Qwen head units). Among equal optima the
           assignment that is smallest in unit order is returned.
   mode 0: Lagrangian allocation with repair (the KDA key-row units): every unit starts at the
           smallest candidate and moves along the lower convex hull of its points (b, J)
           (a middle point is off the hull when its left slope >= its right slope), always
           taking the move with the least (J_next - J_cur)/(b_next - b_cur) that fits the
           remaining bits (ties: lowest unit); leftover bits are then placed by the single
           unit change, or (up, down) pair of two units, that hits the budget with the least
           change of J (ties: singles first, then lowest indices).
   Returns STEPQ_EBUDGET when no assignment reaches the budget. */
STEPQ_API int stepq_allocate_bits(int n_units, int n_cand, const int* cand_host, const double* J_host,
                        int64_t budget_bits, int mode, uint8_t* bits_out_host);

/* Device error word of the library's kernels: bit 0 is set when a bounded wait (for a tile
   copy, or a tensor-core round of the prefill chunk) gave up after its limit (2 s); the kernel
   then waits, bounded, for its own copies in flight, frees its tensor memory and returns, so the
   context stays usable. Bit 1 is set when a width-16 row was met in a launch with
   dims.pivots = 0. Bit 2 is set when a head's byte range in the packed state, [head_off[h],
   head_off[h+1]) (bytes_per_seq for the last head), is unaligned, out of order, outside the
   sequence or shorter than the head's tile under the bit map; the kernels (decode step, prefill
   chunk, split form, pack, unpack) then skip that tile and read or write nothing of it. Reads
   (synchronously, on the current device) and clears it. */
STEPQ_API int stepq_read_device_flags(uint32_t* flags_host);

/* Self-test of that wait limit: one bounded wait that nothing completes (an mbarrier phase no
   thread arrives on), giving up after limit_ns (1e3 to 1e9 ns, else STEPQ_EINVAL before any
   CUDA call) and raising bit 0 of the device error word. Queued on `stream`. */
STEPQ_API int stepq_selftest_wait(uint64_t limit_ns, void* stream);

/* Build description (compute capability compiled for, and version). */
STEPQ_API const char* stepq_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* STEPQ_H */
