/*
 * stepq_oracle.c -- plain CPU oracle for the quantized gated Delta-rule decode step of
 * "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State Quantization".
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path loads this library: only the test
 * suite, the package's smoke check and the benchmark's CPU-baseline leg do. It shares no code,
 * header, table or constant with the CUDA library; the two meet only at the seeded inputs.
 *
 * Precision: the recurrence and every reduction of the scale fit run in double. The
 * quantiser / dequantiser contract, and every step where floating point decides an integer
 * code, run in fp32 exactly as written below (build with -O2 -ffp-contract=off so that no
 * multiply-add is fused). Tiles are processed one at a time by plain loops; the batch loops
 * may run tiles on several threads (OpenMP) and nothing else.
 *
 * What each part follows (sections, equations and tables of the STEPQuant paper):
 *   recurrence        §2.1, the gated Delta rule and its affine form S_t = A_t S_{t-1} + B_t;
 *                     readout y_t = S_t^T q_t taken before requantisation (Table C2, step 3).
 *   gate D_t          scalar per head (GDN) or diagonal over key rows (KDA), §2.1, §6.1 / App. C.1.
 *   quantiser         §2.2, Q_{b,s}(x) = s clip(round(x/s), -q_b, q_b), q_b = 2^(b-1) - 1.
 *   code normalisation App. C.1: stored integer q, reconstruction z = 2^(8-b) q.
 *   dual-axis scales  §4.3, X_hat_ij = r_i c_j z_ij; row factor m_i = mean_j |X_ij| (§4.3
 *                     "Row factors") with the key-row impact factor folded into r_i;
 *                     column fit min_c sum w_i^2 (X_ij - r_i c_j z_ij)^2 (§4.3 "Column
 *                     factors") by the fixed-code closed form of App. C.1 with a positive
 *                     floor and "zero denominator keeps the previous scale".
 *   row impact        App. B.3 / C.1: omega_i = E[(A_t^T q_t)_i^2] with
 *                     (A_t^T q_t)_i = d_i (q_i - beta k_i (k.q)); w_i proportional to omega_i^(1/8).
 *   distortion        App. A.3, Eq. 17 (row-impact-weighted MSE per head) and Eq. 18
 *                     (plain MSE per key row).
 *   bit allocation    §3.2 / App. C.2: multiple-choice dynamic programme (head units) and a
 *                     Lagrangian allocation repaired to the integer budget (row units).
 *   scale metadata    App. D, Eq. 22: fp16 row and column scales, 16(d_k+d_v)/(d_k d_v) bits.
 *
 * Readings where the paper leaves a step open:
 *   R1 r_i = fp16(clamp(max(m_i, 2^-14) / w_i, 2^-14, 65504)).
 *   R2 column initialisation c0_j = max(max_i |X_ij| a_i, 2^-14), a_i = 1/(r_i 2^(8-b_i) q_b),
 *      i.e. the smallest column scale at which no entry clips; then ONE fixed-code
 *      least-squares update over all rows; zero denominator -> c0_j; c_j = fp16(clamp(c1_j)).
 *   R3 quantise: t = (x * ir_i) * ic_j with ir_i = 1/(r_i 2^(8-b_i)), ic_j = 1/c_j, fp32,
 *      q = clamp(rint(t), -q_b, q_b), rint = nearest with ties to even.
 *   R4 dequantise: x_hat = (r_i * c_j) * (float)(q 2^(8-b_i)), fp32.
 *   R5 packed layout: tile (b,h) at b*bytes_per_seq + head_off[h]; row i at
 *      (d_v/8) sum_{i'<i} b_i'; codes are b-bit two's complement. A 2- or 8-bit row stores
 *      the code of column j at bit j*b of a little-endian bit stream. A 4-bit row stores each
 *      group of four columns 4g..4g+3 in the 16-bit little-endian halfword g with the
 *      columns in nibble order (0, 2, 1, 3): column 4g+m sits at bit 4*pos(m),
 *      pos = {0, 2, 1, 3}. A 6-bit row stores the low 4 bits of every code (laid out as a
 *      4-bit row) followed by the high 2 bits (laid out as a 2-bit row).
 *   R6 KDA code normalisation (z = 2^(8-b) q) for every workload.
 *   R7 omega floor 1e-12 max_i omega_i; w normalised to mean 1 per head.
 *   R14 FP16 pivot rows (App. C.2; Table C2 steps 1 and 6), marked by width 16: the row keeps
 *      its values as binary16 (2 d_v bytes, column j at byte 2j, little-endian), stored
 *      after all integer rows of the tile; it takes no part in the shared column fit (c0 and
 *      the least-squares sums run over the integer rows); its row factor is computed like
 *      any other (R1) and is not used.
 *   R15 a pivot value is the fp32 X rounded to binary16, nearest with ties to even,
 *      saturating at +-65504.
 *
 * Parity unpinned: R1's division of the row factor by w_i and R7's use of the 1/8 exponent for
 * KDA rows are readings the paper does not state (it omits the formula, and gives the exponent
 * for Qwen only). The tests pin the definitions around them, such as m_i, omega_i from explicit
 * transition matrices, and the no-clip and least-squares properties of the fit, but not the
 * readings themselves.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_OK = 0, ORC_EINVAL = 1, ORC_EUNSUPPORTED = 2, ORC_EBUDGET = 4, ORC_ENOMEM = 6 };

#define HALF_MIN_NORMAL 0x1p-14
#define HALF_MAX 65504.0

/* ------------------------------------------------------------------------------------------ */
/* Bit widths and codebooks (§2.2, App. C.1).                                                 */
/* ------------------------------------------------------------------------------------------ */

/* b = 16 marks an FP16 pivot row (App. C.2, Table C2 steps 1 and 6; reading R14). */
static int is_pivot(int b) { return b == 16; }
static int width_ok(int b) { return b == 2 || b == 4 || b == 6 || b == 8 || b == 16; }
static int qmax_of(int b) { return (1 << (b - 1)) - 1; }   /* q_b = 2^(b-1) - 1 (integer rows) */
static int znorm_of(int b) { return 1 << (8 - b); }        /* z = 2^(8-b) q       (integer rows) */

int orc_dims_ok(int dk, int dv) { return (dk == 64 || dk == 128) && (dv == 64 || dv == 128); }

/* ------------------------------------------------------------------------------------------ */
/* IEEE 754 binary16 and bfloat16, written from the format definitions.                       */
/* ------------------------------------------------------------------------------------------ */

float orc_half_to_float(uint16_t h) {
    int e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return (float)((h & 0x8000) ? -v : v);
}

float orc_bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* A positive scale rounded to binary16: first clamped into the normal range
   [2^-14, 65504] (NaN goes to the floor), then rounded to nearest, ties to even. */
uint16_t orc_scale_to_half(double x) {
    if (!(x >= HALF_MIN_NORMAL)) x = HALF_MIN_NORMAL;
    if (x > HALF_MAX) x = HALF_MAX;
    int e;
    double m = frexp(x, &e);            /* x = m 2^e, m in [0.5, 1)              */
    double sig = nearbyint(ldexp(m, 11)); /* 11 significant bits, ties to even    */
    if (sig == 2048.0) { sig = 1024.0; e += 1; }
    int E = e - 1 + 15;                  /* binary16 exponent field               */
    return (uint16_t)((E << 10) | ((int)sig - 1024));
}

/* fp32 -> binary16, nearest with ties to even, saturating at +-65504 (reading R15): the value
   stored for an FP16 pivot entry. Written from the binary16 format definition. */
uint16_t orc_float_to_half(float xf) {
    double x = (double)xf;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    x = fabs(x);
    if (isnan(x)) return 0x7E00u;
    if (x > HALF_MAX) return (uint16_t)(sign | 0x7BFFu);
    if (x < HALF_MIN_NORMAL) {                       /* subnormal: steps of 2^-24      */
        double q = nearbyint(ldexp(x, 24));          /* 1024 is 2^-14, the first normal */
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e;
    double m = frexp(x, &e);
    double sig = nearbyint(ldexp(m, 11));
    if (sig == 2048.0) { sig = 1024.0; e += 1; }
    int E = e - 1 + 15;
    if (E >= 31) return (uint16_t)(sign | 0x7BFFu);
    return (uint16_t)(sign | (E << 10) | ((int)sig - 1024));
}

/* ------------------------------------------------------------------------------------------ */
/* Quantiser and dequantiser contract (readings R3, R4), fp32.                                */
/* ------------------------------------------------------------------------------------------ */

static int quantise(float x, float ir, float ic, int b) {
    float t = (x * ir) * ic;
    float n = rintf(t);
    float qb = (float)qmax_of(b);
    if (n > qb) n = qb;
    if (n < -qb) n = -qb;
    return (int)n;
}

static float dequantise(float r, float c, int q, int b) {
    float rc = r * c;
    return rc * (float)(q * znorm_of(b));
}

/* ------------------------------------------------------------------------------------------ */
/* Packed layout (reading R5).                                                                */
/* ------------------------------------------------------------------------------------------ */

static int64_t row_bytes(int dv, int b) { return (int64_t)dv * b / 8; }

int64_t orc_tile_bytes(int dk, int dv, const uint8_t* bits) {
    int64_t n = 0;
    for (int i = 0; i < dk; ++i) n += row_bytes(dv, bits[i]);
    return n;
}

/* Byte offset of every row inside its tile (readings R5, R14): the integer rows first, in key
   order, then the FP16 pivot rows, in key order. */
static void row_offsets(int dk, int dv, const uint8_t* bits, int64_t* off) {
    int64_t o = 0;
    for (int pass = 0; pass < 2; ++pass)
        for (int i = 0; i < dk; ++i)
            if (is_pivot(bits[i]) == pass) {
                off[i] = o;
                o += row_bytes(dv, bits[i]);
            }
}

/* head_off[h] = bytes of heads 0..h-1 of one sequence; returns bytes per sequence. */
int64_t orc_layout(int H, int dk, int dv, const uint8_t* bits, int64_t* head_off) {
    int64_t off = 0;
    for (int h = 0; h < H; ++h) {
        if (head_off) head_off[h] = off;
        off += orc_tile_bytes(dk, dv, bits + (int64_t)h * dk);
    }
    return off;
}

static void put_bits(uint8_t* base, int64_t bitpos, int width, unsigned value) {
    for (int k = 0; k < width; ++k) {
        int64_t p = bitpos + k;
        uint8_t mask = (uint8_t)(1u << (p & 7));
        if ((value >> k) & 1u) base[p >> 3] |= mask;
        else base[p >> 3] &= (uint8_t)~mask;
    }
}

static unsigned get_bits(const uint8_t* base, int64_t bitpos, int width) {
    unsigned v = 0;
    for (int k = 0; k < width; ++k) {
        int64_t p = bitpos + k;
        v |= (unsigned)((base[p >> 3] >> (p & 7)) & 1u) << k;
    }
    return v;
}

/* Bit position of column j inside a row of width b (reading R5). In a 4-bit row the four
   columns of each 16-bit group are kept in nibble order (0, 2, 1, 3). */
static int64_t field_bit(int j, int b) {
    if (b == 4) {
        static const int pos[4] = {0, 2, 1, 3};
        return (int64_t)(j / 4) * 16 + 4 * pos[j % 4];
    }
    return (int64_t)j * b;
}

/* Write the signed codes of one row (dv columns) at width b. */
static void pack_row(uint8_t* row, int dv, int b, const int* q) {
    if (b == 6) {
        uint8_t* lo_plane = row;
        uint8_t* hi_plane = row + dv / 2;
        for (int j = 0; j < dv; ++j) {
            unsigned v = (unsigned)q[j] & 63u;             /* 6-bit two's complement */
            put_bits(lo_plane, field_bit(j, 4), 4, v & 15u);
            put_bits(hi_plane, field_bit(j, 2), 2, v >> 4);
        }
    } else {
        for (int j = 0; j < dv; ++j)
            put_bits(row, field_bit(j, b), b, (unsigned)q[j] & ((1u << b) - 1u));
    }
}

static void unpack_row(const uint8_t* row, int dv, int b, int* q) {
    for (int j = 0; j < dv; ++j) {
        unsigned v;
        if (b == 6) v = get_bits(row, field_bit(j, 4), 4) | (get_bits(row + dv / 2, field_bit(j, 2), 2) << 4);
        else v = get_bits(row, field_bit(j, b), b);
        int s = (int)v;
        if (!is_pivot(b) && s >= (1 << (b - 1))) s -= (1 << b);   /* sign-extend from b bits */
        q[j] = s;                                   /* a pivot entry: its binary16 bit pattern */
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Tile-level operations. X is row-major [dk][dv]: row = key channel, column = value channel. */
/* ------------------------------------------------------------------------------------------ */

/* Codes of a tile at given scales (readings R3, R6). */
void orc_quantise_tile(int dk, int dv, const float* X, const uint8_t* bits, const uint16_t* r,
                       const uint16_t* c, int* codes) {
    for (int i = 0; i < dk; ++i) {
        int b = bits[i];
        if (is_pivot(b)) {                           /* FP16 pivot row: the value itself */
            for (int j = 0; j < dv; ++j) codes[i * dv + j] = orc_float_to_half(X[i * dv + j]);
            continue;
        }
        float ir = 1.0f / (orc_half_to_float(r[i]) * (float)znorm_of(b));
        for (int j = 0; j < dv; ++j) {
            float ic = 1.0f / orc_half_to_float(c[j]);
            codes[i * dv + j] = quantise(X[i * dv + j], ir, ic, b);
        }
    }
}

void orc_pack_codes(int dk, int dv, const uint8_t* bits, const int* codes, uint8_t* packed) {
    int64_t* off = (int64_t*)malloc(sizeof(int64_t) * dk);
    row_offsets(dk, dv, bits, off);
    for (int i = 0; i < dk; ++i) pack_row(packed + off[i], dv, bits[i], codes + (int64_t)i * dv);
    free(off);
}

void orc_unpack_codes(int dk, int dv, const uint8_t* bits, const uint8_t* packed, int* codes) {
    int64_t* off = (int64_t*)malloc(sizeof(int64_t) * dk);
    row_offsets(dk, dv, bits, off);
    for (int i = 0; i < dk; ++i) unpack_row(packed + off[i], dv, bits[i], codes + (int64_t)i * dv);
    free(off);
}

void orc_pack_tile(int dk, int dv, const float* X, const uint8_t* bits, const uint16_t* r,
                   const uint16_t* c, uint8_t* packed) {
    int* codes = (int*)malloc(sizeof(int) * dk * dv);
    orc_quantise_tile(dk, dv, X, bits, r, c, codes);
    orc_pack_codes(dk, dv, bits, codes, packed);
    free(codes);
}

void orc_unpack_tile(int dk, int dv, const uint8_t* packed, const uint8_t* bits, const uint16_t* r,
                     const uint16_t* c, float* X) {
    int* codes = (int*)malloc(sizeof(int) * dk * dv);
    orc_unpack_codes(dk, dv, bits, packed, codes);
    for (int i = 0; i < dk; ++i) {
        float ri = orc_half_to_float(r[i]);
        for (int j = 0; j < dv; ++j)
            X[i * dv + j] = is_pivot(bits[i]) ? orc_half_to_float((uint16_t)codes[i * dv + j])
                                              : dequantise(ri, orc_half_to_float(c[j]), codes[i * dv + j], bits[i]);
    }
    free(codes);
}

/* One fixed-code least-squares update of every column scale (App. C.1) at binary16 row scales
   r and integer codes z [dk][dv]: c_j = sum_i w_i^2 v_ij X_ij / sum_i w_i^2 v_ij^2 with
   v_ij = r_i 2^(8-b_i) z_ij over the non-pivot rows; a column with a zero denominator keeps
   cfall[j]. Returns c as binary16, c1 (double, before rounding) if given. */
void orc_ls_columns(int dk, int dv, const float* X, const float* w, const uint8_t* bits, const uint16_t* r,
                    const int* z, const float* cfall, uint16_t* c_out, double* c1_out) {
    for (int j = 0; j < dv; ++j) {
        double num = 0.0, den = 0.0;
        for (int i = 0; i < dk; ++i) {
            if (is_pivot(bits[i])) continue;
            double v = (double)orc_half_to_float(r[i]) * znorm_of(bits[i]) * z[i * dv + j];
            double ww = (double)w[i] * (double)w[i];
            num += ww * v * (double)X[i * dv + j];
            den += ww * v * v;
        }
        double c1 = den > 0.0 ? num / den : (double)cfall[j];
        if (c1_out) c1_out[j] = c1;
        c_out[j] = orc_scale_to_half(c1);
    }
}

/* The column half of the dual-axis fit (App. C.1; reading R2) at given binary16 row scales r:
   the no-clip column start c0, the codes at (r, c0) and one weighted least-squares update.
   Returns c as binary16; the optional detail outputs expose c0 (fp32), z0 (codes at (r, c0))
   and c1 (double, the least-squares solution before rounding). */
void orc_fit_columns_detail(int dk, int dv, const float* X, const float* w, const uint8_t* bits,
                            const uint16_t* r, uint16_t* c_out, float* c0_out, int* z0_out, double* c1_out) {
    float* rf = (float*)malloc(sizeof(float) * dk);
    float* c0 = (float*)malloc(sizeof(float) * dv);
    int* z0 = (int*)malloc(sizeof(int) * dk * dv);
    for (int i = 0; i < dk; ++i) rf[i] = orc_half_to_float(r[i]);

    /* Column initialisation: smallest scale at which no entry of the column clips. The shared
       column scales serve the integer rows only: FP16 pivot rows take no part (App. C.1, the
       sums over the non-pivot rows I). */
    for (int j = 0; j < dv; ++j) {
        float mx = 0.0f;
        for (int i = 0; i < dk; ++i) {
            int b = bits[i];
            if (is_pivot(b)) continue;
            float a = 1.0f / (rf[i] * (float)(znorm_of(b) * qmax_of(b)));
            float t = fabsf(X[i * dv + j]) * a;
            if (t > mx) mx = t;
        }
        c0[j] = mx < (float)HALF_MIN_NORMAL ? (float)HALF_MIN_NORMAL : mx;
    }

    /* Codes at (r, c0), decided in fp32 by the quantiser contract. */
    for (int i = 0; i < dk; ++i) {
        int b = bits[i];
        if (is_pivot(b)) {
            for (int j = 0; j < dv; ++j) z0[i * dv + j] = 0;
            continue;
        }
        float ir = 1.0f / (rf[i] * (float)znorm_of(b));
        for (int j = 0; j < dv; ++j) z0[i * dv + j] = quantise(X[i * dv + j], ir, 1.0f / c0[j], b);
    }

    orc_ls_columns(dk, dv, X, w, bits, r, z0, c0, c_out, c1_out);
    if (c0_out) memcpy(c0_out, c0, sizeof(float) * dv);
    if (z0_out) memcpy(z0_out, z0, sizeof(int) * dk * dv);
    free(rf);
    free(c0);
    free(z0);
}

/* Key-row-aware dual-axis fit (§4.3, App. C.1; readings R1, R2). Returns r, c as binary16.
   The optional detail outputs are those of orc_fit_columns_detail. */
void orc_fit_tile_detail(int dk, int dv, const float* X, const float* w, const uint8_t* bits,
                         uint16_t* r_out, uint16_t* c_out, float* c0_out, int* z0_out,
                         double* c1_out) {
    /* Row factors: m_i = (1/d_v) sum_j |X_ij|, impact folded in as r_i = m_i / w_i. */
    for (int i = 0; i < dk; ++i) {
        double m = 0.0;
        for (int j = 0; j < dv; ++j) m += fabs((double)X[i * dv + j]);
        m /= dv;
        if (m < HALF_MIN_NORMAL) m = HALF_MIN_NORMAL;
        r_out[i] = orc_scale_to_half(m / (double)w[i]);
    }
    orc_fit_columns_detail(dk, dv, X, w, bits, r_out, c_out, c0_out, z0_out, c1_out);
}

void orc_fit_tile(int dk, int dv, const float* X, const float* w, const uint8_t* bits,
                  uint16_t* r_out, uint16_t* c_out) {
    orc_fit_tile_detail(dk, dv, X, w, bits, r_out, c_out, NULL, NULL, NULL);
}

/* One gated Delta-rule update in double (§2.1):
     X = D S + beta k (v^T - k^T D S),  o = X^T q.
   gate has dk entries (the diagonal of D; a scalar gate is repeated). */
void orc_delta_update(int dk, int dv, const double* S, const double* q, const double* k,
                      const double* v, double beta, const double* gate, double* X, double* o) {
    double* p = (double*)calloc(dv, sizeof(double));
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) X[i * dv + j] = gate[i] * S[i * dv + j];
    for (int j = 0; j < dv; ++j)
        for (int i = 0; i < dk; ++i) p[j] += k[i] * X[i * dv + j];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) X[i * dv + j] += k[i] * (beta * (v[j] - p[j]));
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += q[i] * X[i * dv + j];
        o[j] = acc;
    }
    free(p);
}

typedef struct {
    int dk, dv;
    double *q, *k, *v, *g, *S, *X, *o;
} orc_tile_scratch;

static void tile_inputs(orc_tile_scratch* t, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const float* gate, int gate_per_channel) {
    for (int i = 0; i < t->dk; ++i) {
        t->q[i] = orc_bf16_to_float(q[i]);
        t->k[i] = orc_bf16_to_float(k[i]);
        t->g[i] = gate_per_channel ? (double)gate[i] : (double)gate[0];
    }
    for (int j = 0; j < t->dv; ++j) t->v[j] = orc_bf16_to_float(v[j]);
}

static int scratch_alloc(orc_tile_scratch* t, int dk, int dv) {
    t->dk = dk;
    t->dv = dv;
    t->q = (double*)malloc(sizeof(double) * dk);
    t->k = (double*)malloc(sizeof(double) * dk);
    t->g = (double*)malloc(sizeof(double) * dk);
    t->v = (double*)malloc(sizeof(double) * dv);
    t->o = (double*)malloc(sizeof(double) * dv);
    t->S = (double*)malloc(sizeof(double) * dk * dv);
    t->X = (double*)malloc(sizeof(double) * dk * dv);
    return t->q && t->k && t->g && t->v && t->o && t->S && t->X;
}

static void scratch_free(orc_tile_scratch* t) {
    free(t->q); free(t->k); free(t->g); free(t->v); free(t->o); free(t->S); free(t->X);
}

/* One persistent decode step of one tile (Table C2): reconstruct the previous state from
   codes and scales, apply the gated Delta update, emit the readout before requantisation,
   refit the dual-axis scales on the updated state and repack it. */
void orc_decode_tile(int dk, int dv, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     float beta, const float* gate, int gate_per_channel, const uint8_t* bits,
                     const float* w, const uint8_t* packed_in, const uint16_t* r_in,
                     const uint16_t* c_in, uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out,
                     float* o) {
    orc_tile_scratch t;
    scratch_alloc(&t, dk, dv);
    float* S32 = (float*)malloc(sizeof(float) * dk * dv);
    tile_inputs(&t, q, k, v, gate, gate_per_channel);
    orc_unpack_tile(dk, dv, packed_in, bits, r_in, c_in, S32);                 /* step 1 */
    for (int e = 0; e < dk * dv; ++e) t.S[e] = S32[e];
    orc_delta_update(dk, dv, t.S, t.q, t.k, t.v, (double)beta, t.g, t.X, t.o); /* step 2 */
    for (int j = 0; j < dv; ++j) o[j] = (float)t.o[j];                         /* step 3 */
    for (int e = 0; e < dk * dv; ++e) S32[e] = (float)t.X[e];
    orc_fit_tile(dk, dv, S32, w, bits, r_out, c_out);                          /* steps 4-5 */
    orc_pack_tile(dk, dv, S32, bits, r_out, c_out, packed_out);                /* step 6 */
    free(S32);
    scratch_free(&t);
}

/* FP32-state decode step (the unquantised baseline state format, §5.1). */
void orc_decode_tile_fp32(int dk, int dv, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          float beta, const float* gate, int gate_per_channel, const float* S_in,
                          float* S_out, float* o) {
    orc_tile_scratch t;
    scratch_alloc(&t, dk, dv);
    tile_inputs(&t, q, k, v, gate, gate_per_channel);
    for (int e = 0; e < dk * dv; ++e) t.S[e] = S_in[e];
    orc_delta_update(dk, dv, t.S, t.q, t.k, t.v, (double)beta, t.g, t.X, t.o);
    for (int j = 0; j < dv; ++j) o[j] = (float)t.o[j];
    for (int e = 0; e < dk * dv; ++e) S_out[e] = (float)t.X[e];
    scratch_free(&t);
}

/* Symmetric rowwise-absmax INT8 state (the uniform baseline of §5.1): x_hat = s_i q,
   s_i = fp16(max_j |X_ij| / 127), q = clamp(rint(X * (1/s_i)), -127, 127). */
void orc_int8_quantise_tile(int dk, int dv, const float* X, int8_t* codes, uint16_t* s) {
    for (int i = 0; i < dk; ++i) {
        float mx = 0.0f;
        for (int j = 0; j < dv; ++j) if (fabsf(X[i * dv + j]) > mx) mx = fabsf(X[i * dv + j]);
        s[i] = orc_scale_to_half((double)mx / 127.0);
        float is = 1.0f / orc_half_to_float(s[i]);
        for (int j = 0; j < dv; ++j) {
            float n = rintf(X[i * dv + j] * is);
            if (n > 127.0f) n = 127.0f;
            if (n < -127.0f) n = -127.0f;
            codes[i * dv + j] = (int8_t)n;
        }
    }
}

void orc_decode_tile_int8(int dk, int dv, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          float beta, const float* gate, int gate_per_channel, const int8_t* codes_in,
                          const uint16_t* s_in, int8_t* codes_out, uint16_t* s_out, float* o) {
    orc_tile_scratch t;
    scratch_alloc(&t, dk, dv);
    float* S32 = (float*)malloc(sizeof(float) * dk * dv);
    tile_inputs(&t, q, k, v, gate, gate_per_channel);
    for (int i = 0; i < dk; ++i) {
        float si = orc_half_to_float(s_in[i]);
        for (int j = 0; j < dv; ++j) t.S[i * dv + j] = (double)(si * (float)codes_in[i * dv + j]);
    }
    orc_delta_update(dk, dv, t.S, t.q, t.k, t.v, (double)beta, t.g, t.X, t.o);
    for (int j = 0; j < dv; ++j) o[j] = (float)t.o[j];
    for (int e = 0; e < dk * dv; ++e) S32[e] = (float)t.X[e];
    orc_int8_quantise_tile(dk, dv, S32, codes_out, s_out);
    free(S32);
    scratch_free(&t);
}

/* ------------------------------------------------------------------------------------------ */
/* Batch loops over (sequence b, head h) tiles. Arrays are [B][H][...] row-major; the packed  */
/* state of tile (b,h) starts at b*bytes_per_seq + head_off[h].                              */
/* ------------------------------------------------------------------------------------------ */

static int set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    return nthreads;
#else
    (void)nthreads;
    return 1;
#endif
}

int orc_fit_scales(int B, int H, int dk, int dv, const float* S, const float* w, const uint8_t* bits,
                   uint16_t* r, uint16_t* c, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t t = 0; t < n; ++t) {
        int h = (int)(t % H);
        orc_fit_tile(dk, dv, S + t * dk * dv, w + (int64_t)h * dk, bits + (int64_t)h * dk,
                     r + t * dk, c + t * dv);
    }
    return ORC_OK;
}

int orc_pack_state(int B, int H, int dk, int dv, const float* S, const uint8_t* bits,
                   const int64_t* head_off, int64_t bytes_per_seq, const uint16_t* r,
                   const uint16_t* c, uint8_t* packed, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t t = 0; t < n; ++t) {
        int64_t b = t / H;
        int h = (int)(t % H);
        orc_pack_tile(dk, dv, S + t * dk * dv, bits + (int64_t)h * dk, r + t * dk, c + t * dv,
                      packed + b * bytes_per_seq + head_off[h]);
    }
    return ORC_OK;
}

int orc_unpack_state(int B, int H, int dk, int dv, const uint8_t* packed, const uint8_t* bits,
                     const int64_t* head_off, int64_t bytes_per_seq, const uint16_t* r,
                     const uint16_t* c, float* S, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t t = 0; t < n; ++t) {
        int64_t b = t / H;
        int h = (int)(t % H);
        orc_unpack_tile(dk, dv, packed + b * bytes_per_seq + head_off[h], bits + (int64_t)h * dk,
                        r + t * dk, c + t * dv, S + t * dk * dv);
    }
    return ORC_OK;
}

int orc_decode_step(int B, int H, int dk, int dv, int gate_per_channel, const uint16_t* q,
                    const uint16_t* k, const uint16_t* v, const float* beta, const float* gate,
                    const uint8_t* bits, const float* w, const int64_t* head_off,
                    int64_t bytes_per_seq, const uint8_t* packed_in, const uint16_t* r_in,
                    const uint16_t* c_in, uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out,
                    float* o, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    int gstride = gate_per_channel ? dk : 1;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t t = 0; t < n; ++t) {
        int64_t b = t / H;
        int h = (int)(t % H);
        int64_t off = b * bytes_per_seq + head_off[h];
        orc_decode_tile(dk, dv, q + t * dk, k + t * dk, v + t * dv, beta[t], gate + t * gstride,
                        gate_per_channel, bits + (int64_t)h * dk, w + (int64_t)h * dk,
                        packed_in + off, r_in + t * dk, c_in + t * dv, packed_out + off,
                        r_out + t * dk, c_out + t * dv, o + t * dv);
    }
    return ORC_OK;
}

/* A prefill chunk of C tokens on the packed state (App. F.1: the native chunk update runs on
   the unpacked state and the boundary state is packed once; App. B.2): reconstruct S_hat,
   apply the gated Delta rule C times in double (each readout o_t = X_t^T q_t), then fit and
   pack the final state once. Inputs carry a leading token axis: q, k [C][B][H][dk], v
   [C][B][H][dv], beta [C][B][H], gate [C][B][H] or [C][B][H][dk]; o [C][B][H][dv]. */
int orc_prefill_chunk(int C, int B, int H, int dk, int dv, int gate_per_channel, const uint16_t* q,
                      const uint16_t* k, const uint16_t* v, const float* beta, const float* gate,
                      const uint8_t* bits, const float* w, const int64_t* head_off,
                      int64_t bytes_per_seq, const uint8_t* packed_in, const uint16_t* r_in,
                      const uint16_t* c_in, uint8_t* packed_out, uint16_t* r_out, uint16_t* c_out,
                      float* o, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    if (C < 1) return ORC_EINVAL;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    int gstride = gate_per_channel ? dk : 1;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t tl = 0; tl < n; ++tl) {
        int64_t b = tl / H;
        int h = (int)(tl % H);
        int64_t off = b * bytes_per_seq + head_off[h];
        const uint8_t* bh = bits + (int64_t)h * dk;
        orc_tile_scratch t;
        scratch_alloc(&t, dk, dv);
        float* S32 = (float*)malloc(sizeof(float) * dk * dv);
        orc_unpack_tile(dk, dv, packed_in + off, bh, r_in + tl * dk, c_in + tl * dv, S32);
        for (int e = 0; e < dk * dv; ++e) t.S[e] = S32[e];
        for (int c = 0; c < C; ++c) {
            int64_t tc = (int64_t)c * n + tl;
            tile_inputs(&t, q + tc * dk, k + tc * dk, v + tc * dv, gate + tc * gstride, gate_per_channel);
            orc_delta_update(dk, dv, t.S, t.q, t.k, t.v, (double)beta[tc], t.g, t.X, t.o);
            for (int j = 0; j < dv; ++j) o[tc * dv + j] = (float)t.o[j];
            memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* full precision in between */
        }
        for (int e = 0; e < dk * dv; ++e) S32[e] = (float)t.X[e];
        orc_fit_tile(dk, dv, S32, w + (int64_t)h * dk, bh, r_out + tl * dk, c_out + tl * dv);
        orc_pack_tile(dk, dv, S32, bh, r_out + tl * dk, c_out + tl * dv, packed_out + off);
        free(S32);
        scratch_free(&t);
    }
    return ORC_OK;
}

/* Per-window 8-bit state (LeapQuant, as its abstract on the page "When Dynamic Scaling Fails: A
   Scale-State Feedback Governs Recurrent-State Quantization in Linear-Attention and SSM LLMs"
   describes it: the state is quantised once at the end of a window of tokens; inside the window,
   readouts come from the fixed low-bit state together with high-precision buffered updates). Reading: the
   state between windows is the rowwise-absmax INT8 format of §5.1 (orc_int8_quantise_tile); a
   window of W tokens applies the gated Delta rule exactly (float64) to the reconstructed state
   S_hat = diag(s) codes, every token's readout taken from that running state (which is what the
   fixed state plus the buffered updates equal), and the window's final state is quantised once.
   Token inputs carry a leading token axis of B*H tiles each, like orc_prefill_chunk. */
int orc_leap_window(int W, int B, int H, int dk, int dv, int gate_per_channel, const uint16_t* q,
                    const uint16_t* k, const uint16_t* v, const float* beta, const float* gate,
                    const int8_t* codes_in, const uint16_t* s_in, int8_t* codes_out, uint16_t* s_out,
                    float* o, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    if (W < 1) return ORC_EINVAL;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    int gstride = gate_per_channel ? dk : 1;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t tl = 0; tl < n; ++tl) {
        orc_tile_scratch t;
        scratch_alloc(&t, dk, dv);
        float* S32 = (float*)malloc(sizeof(float) * dk * dv);
        for (int i = 0; i < dk; ++i) {
            float si = orc_half_to_float(s_in[tl * dk + i]);
            for (int j = 0; j < dv; ++j) t.S[i * dv + j] = (double)(si * (float)codes_in[(tl * dk + i) * dv + j]);
        }
        for (int c = 0; c < W; ++c) {
            int64_t tc = (int64_t)c * n + tl;
            tile_inputs(&t, q + tc * dk, k + tc * dk, v + tc * dv, gate + tc * gstride, gate_per_channel);
            orc_delta_update(dk, dv, t.S, t.q, t.k, t.v, (double)beta[tc], t.g, t.X, t.o);
            for (int j = 0; j < dv; ++j) o[tc * dv + j] = (float)t.o[j];
            memcpy(t.S, t.X, sizeof(double) * dk * dv);            /* no quantisation inside the window */
        }
        for (int e = 0; e < dk * dv; ++e) S32[e] = (float)t.X[e];
        orc_int8_quantise_tile(dk, dv, S32, codes_out + tl * dk * dv, s_out + tl * dk);
        free(S32);
        scratch_free(&t);
    }
    return ORC_OK;
}

int orc_decode_step_fp32(int B, int H, int dk, int dv, int gate_per_channel, const uint16_t* q,
                         const uint16_t* k, const uint16_t* v, const float* beta, const float* gate,
                         const float* S_in, float* S_out, float* o, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    int gstride = gate_per_channel ? dk : 1;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t t = 0; t < n; ++t)
        orc_decode_tile_fp32(dk, dv, q + t * dk, k + t * dk, v + t * dv, beta[t], gate + t * gstride,
                             gate_per_channel, S_in + t * dk * dv, S_out + t * dk * dv, o + t * dv);
    return ORC_OK;
}

int orc_decode_step_int8(int B, int H, int dk, int dv, int gate_per_channel, const uint16_t* q,
                         const uint16_t* k, const uint16_t* v, const float* beta, const float* gate,
                         const int8_t* codes_in, const uint16_t* s_in, int8_t* codes_out,
                         uint16_t* s_out, float* o, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    int64_t n = (int64_t)B * H;
    int gstride = gate_per_channel ? dk : 1;
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t t = 0; t < n; ++t)
        orc_decode_tile_int8(dk, dv, q + t * dk, k + t * dk, v + t * dv, beta[t], gate + t * gstride,
                             gate_per_channel, codes_in + t * dk * dv, s_in + t * dk,
                             codes_out + t * dk * dv, s_out + t * dk, o + t * dv);
    return ORC_OK;
}

int orc_int8_quantise_state(int B, int H, int dk, int dv, const float* S, int8_t* codes, uint16_t* s) {
    int64_t n = (int64_t)B * H;
    for (int64_t t = 0; t < n; ++t) orc_int8_quantise_tile(dk, dv, S + t * dk * dv, codes + t * dk * dv, s + t * dk);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Offline calibration (App. A.3, B.3, C.1, C.2).                                            */
/* ------------------------------------------------------------------------------------------ */

/* Row impact over a calibration stream of T steps:
   omega_{h,i} = mean over (t, b) of (d_{t,i} [q_{t,i} - beta_t k_{t,i} (k_t . q_t)])^2,
   floored at 1e-12 max_i omega_{h,i}; w_{h,i} = omega^(1/8) normalised to mean 1 per head. */
int orc_row_impact(int T, int B, int H, int dk, int gate_per_channel, const uint16_t* q,
                   const uint16_t* k, const float* beta, const float* gate, float* w_out) {
    double* om = (double*)calloc((size_t)H * dk, sizeof(double));
    if (!om) return ORC_ENOMEM;
    int gstride = gate_per_channel ? dk : 1;
    for (int t = 0; t < T; ++t)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h) {
                int64_t tile = ((int64_t)t * B + b) * H + h;
                const uint16_t* qq = q + tile * dk;
                const uint16_t* kk = k + tile * dk;
                double kq = 0.0;
                for (int i = 0; i < dk; ++i) kq += (double)orc_bf16_to_float(kk[i]) * orc_bf16_to_float(qq[i]);
                for (int i = 0; i < dk; ++i) {
                    double d = gate_per_channel ? gate[tile * gstride + i] : gate[tile * gstride];
                    double g = d * (orc_bf16_to_float(qq[i]) - (double)beta[tile] * orc_bf16_to_float(kk[i]) * kq);
                    om[(int64_t)h * dk + i] += g * g;
                }
            }
    for (int h = 0; h < H; ++h) {
        double* oh = om + (int64_t)h * dk;
        double mx = 0.0, mean = 0.0;
        for (int i = 0; i < dk; ++i) { oh[i] /= (double)T * B; if (oh[i] > mx) mx = oh[i]; }
        for (int i = 0; i < dk; ++i) {
            if (oh[i] < 1e-12 * mx) oh[i] = 1e-12 * mx;
            oh[i] = pow(oh[i], 0.125);
            mean += oh[i];
        }
        mean /= dk;
        for (int i = 0; i < dk; ++i) w_out[(int64_t)h * dk + i] = (float)(mean > 0.0 ? oh[i] / mean : 1.0);
    }
    free(om);
    return ORC_OK;
}

/* Candidate-format distortion of the B sample states under the bit map bits [H][dk]
   (App. A.3): d_row[h][i] = (1/(B d_v)) sum_b sum_j (x_hat - x)^2                (Eq. 18)
               d_head[h]   = (1/(B d_k d_v)) sum_b sum_ij w_i^2 (x_hat - x)^2      (Eq. 17)
   where x_hat is the state fitted, packed and unpacked under that map. */
int orc_calib_distortion_bits(int B, int H, int dk, int dv, const float* S, const float* w,
                              const uint8_t* bits_map, double* d_row, double* d_head, int nthreads) {
    if (!orc_dims_ok(dk, dv)) return ORC_EUNSUPPORTED;
    for (int64_t u = 0; u < (int64_t)H * dk; ++u)
        if (!width_ok(bits_map[u])) return ORC_EUNSUPPORTED;
    int nt = set_threads(nthreads);
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int h = 0; h < H; ++h) {
        const uint8_t* bits = bits_map + (int64_t)h * dk;
        uint16_t* r = (uint16_t*)malloc(sizeof(uint16_t) * dk);
        uint16_t* c = (uint16_t*)malloc(sizeof(uint16_t) * dv);
        uint8_t* pk = (uint8_t*)malloc(orc_tile_bytes(dk, dv, bits));
        float* Xh = (float*)malloc(sizeof(float) * dk * dv);
        double dh = 0.0;
        for (int i = 0; i < dk; ++i) d_row[(int64_t)h * dk + i] = 0.0;
        for (int s = 0; s < B; ++s) {
            const float* X = S + ((int64_t)s * H + h) * dk * dv;
            const float* wh = w + (int64_t)h * dk;
            orc_fit_tile(dk, dv, X, wh, bits, r, c);
            orc_pack_tile(dk, dv, X, bits, r, c, pk);
            orc_unpack_tile(dk, dv, pk, bits, r, c, Xh);
            for (int i = 0; i < dk; ++i) {
                double row = 0.0;
                for (int j = 0; j < dv; ++j) {
                    double e = (double)Xh[i * dv + j] - (double)X[i * dv + j];
                    row += e * e;
                }
                d_row[(int64_t)h * dk + i] += row;
                dh += (double)wh[i] * (double)wh[i] * row;
            }
        }
        for (int i = 0; i < dk; ++i) d_row[(int64_t)h * dk + i] /= (double)B * dv;
        d_head[h] = dh / ((double)B * dk * dv);
        free(r); free(c); free(pk); free(Xh);
    }
    return ORC_OK;
}

/* The same at the uniform width b (every row of every head). */
int orc_calib_distortion(int B, int H, int dk, int dv, const float* S, const float* w, int b,
                         double* d_row, double* d_head, int nthreads) {
    if (!orc_dims_ok(dk, dv) || !width_ok(b)) return ORC_EUNSUPPORTED;
    uint8_t* bits = (uint8_t*)malloc((size_t)H * dk);
    memset(bits, b, (size_t)H * dk);
    int rc = orc_calib_distortion_bits(B, H, dk, dv, S, w, bits, d_row, d_head, nthreads);
    free(bits);
    return rc;
}

/* ------------------------------------------------------------------------------------------ */
/* Lifetime-aware bit allocation (§3.2, App. C.2). J[u][k] is the objective of unit u at      */
/* candidate width cand[k] (ascending). The allocation uses exactly budget bits.              */
/* ------------------------------------------------------------------------------------------ */

/* Multiple-choice dynamic programme, written backwards: G[u][s] is the least cost of units
   u..n-1 using exactly s bits. The assignment is rebuilt from unit 0 on, each unit taking the
   smallest candidate that attains G[u][s]. */
static int alloc_dp(int n, int nc, const int* cand, const double* J, int64_t budget, uint8_t* out) {
    int64_t W = budget + 1;
    if ((double)(n + 1) * (double)W > 6.0e7) return ORC_EINVAL;
    double* G = (double*)malloc(sizeof(double) * (size_t)(n + 1) * (size_t)W);
    if (!G) return ORC_ENOMEM;
    for (int64_t s = 0; s < W; ++s) G[(int64_t)n * W + s] = (s == 0) ? 0.0 : INFINITY;
    for (int u = n - 1; u >= 0; --u)
        for (int64_t s = 0; s < W; ++s) {
            double best = INFINITY;
            for (int kk = 0; kk < nc; ++kk) {
                int64_t rest = s - cand[kk];
                if (rest < 0) continue;
                double nxt = G[(int64_t)(u + 1) * W + rest];
                if (isinf(nxt)) continue;
                double val = J[(int64_t)u * nc + kk] + nxt;
                if (val < best) best = val;
            }
            G[(int64_t)u * W + s] = best;
        }
    if (isinf(G[budget])) { free(G); return ORC_EBUDGET; }
    int64_t s = budget;
    for (int u = 0; u < n; ++u) {
        int chosen = -1;
        for (int kk = 0; kk < nc && chosen < 0; ++kk) {
            int64_t rest = s - cand[kk];
            if (rest < 0) continue;
            double nxt = G[(int64_t)(u + 1) * W + rest];
            if (isinf(nxt)) continue;
            if (J[(int64_t)u * nc + kk] + nxt == G[(int64_t)u * W + s]) chosen = kk;
        }
        out[u] = (uint8_t)cand[chosen];
        s -= cand[chosen];
    }
    free(G);
    return ORC_OK;
}

/* Lagrangian allocation with repair. Each unit walks along the lower convex hull of its
   points (cand_k, J_uk): vertex p1 between p0 and p2 is dropped when
   slope(p0,p1) >= slope(p1,p2). All units start at the smallest candidate; then, while some
   unit's next hull vertex fits the remaining budget, the move with the smallest
   (J_next - J_cur) / (b_next - b_cur) is taken (ties: lowest unit index). If bits remain,
   one repair move reaches the budget exactly: a single unit change by the remainder, or a
   pair (one unit up, another down) whose net change is the remainder, whichever changes J
   least (ties: singles before pairs, then lowest indices in (u, v, new_u, new_v) order). */
static int alloc_lagrange(int n, int nc, const int* cand, const double* J, int64_t budget,
                          uint8_t* out) {
    int* hull = (int*)malloc(sizeof(int) * (size_t)n * nc);
    int* hlen = (int*)malloc(sizeof(int) * n);
    int* pos = (int*)malloc(sizeof(int) * n);
    int* cur = (int*)malloc(sizeof(int) * n); /* candidate index */
    if (!hull || !hlen || !pos || !cur) { free(hull); free(hlen); free(pos); free(cur); return ORC_ENOMEM; }
    int64_t used = 0;
    for (int u = 0; u < n; ++u) {
        const double* Ju = J + (int64_t)u * nc;
        int* hu = hull + (int64_t)u * nc;
        int m = 0;
        for (int kk = 0; kk < nc; ++kk) {
            while (m >= 2) {
                int a = hu[m - 2], b = hu[m - 1];
                double s1 = (Ju[b] - Ju[a]) / (double)(cand[b] - cand[a]);
                double s2 = (Ju[kk] - Ju[b]) / (double)(cand[kk] - cand[b]);
                if (s1 >= s2) --m; else break;
            }
            hu[m++] = kk;
        }
        hlen[u] = m;
        pos[u] = 0;
        cur[u] = hu[0];
        used += cand[hu[0]];
    }
    int64_t rem = budget - used;
    int rc = ORC_OK;
    if (rem < 0) { rc = ORC_EBUDGET; goto done; }
    for (;;) {
        int best = -1;
        double best_slope = 0.0;
        for (int u = 0; u < n; ++u) {
            if (pos[u] + 1 >= hlen[u]) continue;
            int a = hull[(int64_t)u * nc + pos[u]], b = hull[(int64_t)u * nc + pos[u] + 1];
            int64_t db = cand[b] - cand[a];
            if (db > rem) continue;
            double slope = (J[(int64_t)u * nc + b] - J[(int64_t)u * nc + a]) / (double)db;
            if (best < 0 || slope < best_slope) { best = u; best_slope = slope; }
        }
        if (best < 0) break;
        int a = hull[(int64_t)best * nc + pos[best]], b = hull[(int64_t)best * nc + pos[best] + 1];
        rem -= cand[b] - cand[a];
        pos[best] += 1;
        cur[best] = b;
    }
    if (rem > 0) {
        int found = 0, bu = -1, bv = -1, bku = -1, bkv = -1;
        double bdj = 0.0;
        for (int u = 0; u < n; ++u)            /* single moves */
            for (int kk = 0; kk < nc; ++kk) {
                if (cand[kk] - cand[cur[u]] != rem) continue;
                double dj = J[(int64_t)u * nc + kk] - J[(int64_t)u * nc + cur[u]];
                if (!found || dj < bdj) { found = 1; bdj = dj; bu = u; bku = kk; bv = -1; }
            }
        for (int u = 0; u < n; ++u)            /* (up, down) pairs */
            for (int v = 0; v < n; ++v) {
                if (v == u) continue;
                for (int ku = 0; ku < nc; ++ku) {
                    int64_t up = cand[ku] - cand[cur[u]];
                    if (up <= 0) continue;
                    for (int kv = 0; kv < nc; ++kv) {
                        int64_t down = cand[cur[v]] - cand[kv];
                        if (down <= 0 || up - down != rem) continue;
                        double dj = (J[(int64_t)u * nc + ku] - J[(int64_t)u * nc + cur[u]]) +
                                    (J[(int64_t)v * nc + kv] - J[(int64_t)v * nc + cur[v]]);
                        if (!found || dj < bdj) { found = 1; bdj = dj; bu = u; bku = ku; bv = v; bkv = kv; }
                    }
                }
            }
        if (!found) { rc = ORC_EBUDGET; goto done; }
        cur[bu] = bku;
        if (bv >= 0) cur[bv] = bkv;
    }
    for (int u = 0; u < n; ++u) out[u] = (uint8_t)cand[cur[u]];
done:
    free(hull); free(hlen); free(pos); free(cur);
    return rc;
}

int orc_allocate_bits(int n_units, int n_cand, const int* cand, const double* J, int64_t budget,
                      int mode, uint8_t* bits_out) {
    if (n_units <= 0 || n_cand <= 0 || !cand || !J || !bits_out) return ORC_EINVAL;
    for (int kk = 0; kk < n_cand; ++kk) {
        if (cand[kk] <= 0 || cand[kk] > 16) return ORC_EINVAL;
        if (kk > 0 && cand[kk] <= cand[kk - 1]) return ORC_EINVAL;
    }
    if (mode == 1) return alloc_dp(n_units, n_cand, cand, J, budget, bits_out);
    if (mode == 0) return alloc_lagrange(n_units, n_cand, cand, J, budget, bits_out);
    return ORC_EINVAL;
}
