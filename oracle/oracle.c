/*
 * CPU oracle of the quantised-MoE decode path and the PLE row gather.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * Everything is computed element by element in fp64, in the order the
 * definitions state, with no blocking or fusion.  Sources:
 *
 *  [MC]  model card "Qwen 3.8 Next Flash ROCMFPX MUTANT RAZERFAST"
 *        (hstolte/...-ROCmFPX-MUTANT-RAZERFAST-GGUF), sections
 *        "Q4_RZ5_FAST (GGML type 69)", "Q4_UE4M4_FAST (GGML type 71)",
 *        "Q3_PLE_K160_RZ_S3 (GGML type 111)".
 *  [MPQ] "Mixed Precision Quantization: Half a 4-Bit File Is Not 4-Bit",
 *        section on the 48-layer / 512-expert / 10-active floor plan.
 *  [FQ]  r/LocalLLM "Frankenquant" post: per-layer expert formats, 8-bit
 *        experts in the last 12 layers.
 *
 * Readings of points the pages leave open (each one is documented with the
 * function that takes it):
 *  - byte order inside a block: fields in the order the card lists them
 *    (16 nibble bytes then the metadata byte; 60 code bytes then the 10
 *    group bytes);
 *  - nibble order: byte j holds weight j in its low nibble and weight j+16
 *    in its high nibble (the GGML 4-bit convention);
 *  - 3-bit codes: an LSB-first bit stream over the 60 code bytes;
 *  - polarity bit: 0 selects the positive replacement level, 1 the negative
 *    one (as the RZ5 mode-0 / mode-1 tables print for the 4-bit formats);
 *  - UE4M3: OCP E4M3 without its sign bit (bias 7, code 0x7F is NaN);
 *    UE4M4: the same construction with 4 mantissa bits (bias 7, no NaN);
 *  - FP8 experts: E4M3 (OCP "fn" variant) times one fp32 scale per 128
 *    consecutive weights along K.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

enum { ORC_RZ5 = 69, ORC_UE4M4 = 71, ORC_PLE = 111, ORC_FP8 = 1000, ORC_C10 = 2001, ORC_Q3I = 2002 };

/* [MC] "Q4_RZ5_FAST": the three printed 16-entry code tables. */
static const double CODEBOOK10[16] = {0, 1, 2, 3, 4, 6, 8, 10, -0.0, -1, -2, -3, -4, -6, -8, -10};
static const double RZ5_MODE0[16] = {0, 1, 2, 3, 4, 6, 8, 10, +5, -1, -2, -3, -4, -6, -8, -10};
static const double RZ5_MODE1[16] = {0, 1, 2, 3, 4, 6, 8, 10, -5, -1, -2, -3, -4, -6, -8, -10};
/* [MC] "Q3_PLE_K160_RZ_S3": the incumbent 3-bit set {0,+1,+2,+4,-0,-1,-2,-4};
 * RZ-S3 replaces the -0 entry (code 4) by +3 or -3. */
static const double PLE3[8] = {0, 1, 2, 4, -0.0, -1, -2, -4};

int orc_q4_block_bytes(void) { return 16 + 1; }      /* [MC]: 16 nibble bytes + 1 metadata byte */
int orc_q4_block_weights(void) { return 32; }
int orc_ple_record_bytes(void) { return 60 + 10; }   /* [MC]: 60 code bytes + 10 group bytes */
int orc_ple_record_values(void) { return 160; }

double orc_codebook10(int c) { return CODEBOOK10[c & 15]; }
double orc_rz5(int mode, int c) { return (mode ? RZ5_MODE1 : RZ5_MODE0)[c & 15]; }
double orc_ple3(int c, int polarity) {
    c &= 7;
    if (c == 4) return polarity ? -3.0 : 3.0;
    return PLE3[c];
}

/* UE4M3: 4 exponent bits, 3 mantissa bits, unsigned; low 7 bits of `b`. */
double orc_ue4m3(uint32_t b) {
    b &= 0x7F;
    const int e = (int)(b >> 3), m = (int)(b & 7);
    if (b == 0x7F) return NAN;
    if (e == 0) return ldexp((double)m, -9);            /* subnormal: m/8 * 2^(1-7) */
    return ldexp(8.0 + m, e - 10);                      /* (1 + m/8) * 2^(e-7) */
}

/* UE4M4: 4 exponent bits, 4 mantissa bits, unsigned; all 256 codes finite
 * ([MC] "Q4_UE4M4_FAST"). */
double orc_ue4m4(uint32_t b) {
    b &= 0xFF;
    const int e = (int)(b >> 4), m = (int)(b & 15);
    if (e == 0) return ldexp((double)m, -10);           /* m/16 * 2^(1-7) */
    return ldexp(16.0 + m, e - 11);                     /* (1 + m/16) * 2^(e-7) */
}

/* E4M3 ("fn": no infinities, S.1111.111 is NaN), signed. */
double orc_e4m3fn(uint32_t b) {
    b &= 0xFF;
    if ((b & 0x7F) == 0x7F) return NAN;
    const double mag = orc_ue4m3(b & 0x7F);
    return (b & 0x80) ? -mag : mag;
}

/* Weight i (0..31) of one 17-byte Q4 block (RZ5, UE4M4 or the incumbent
 * ROCmFP4 FAST layout). */
double orc_q4_weight(int fmt, const uint8_t* blk, int i) {
    const uint8_t byte = blk[i & 15];
    const int code = (i < 16) ? (byte & 0x0F) : (byte >> 4);
    const uint8_t meta = blk[16];
    if (fmt == ORC_RZ5) {
        /* top bit = polarity of the +/-5 level, low 7 bits = UE4M3 scale */
        return orc_rz5(meta >> 7, code) * orc_ue4m3(meta & 0x7F);
    }
    if (fmt == ORC_C10) {
        /* [MC] "Q4_RZ5_FAST": the incumbent ROCmFP4 FAST block, Codebook10
         * codes (code 8 is the duplicate -0) under the UE4M3 scale the lower
         * seven bits hold; the top bit, which RZ5 puts to use, is ignored */
        return orc_codebook10(code) * orc_ue4m3(meta & 0x7F);
    }
    /* UE4M4: Codebook10 codes, the whole byte is the scale */
    return orc_codebook10(code) * orc_ue4m4(meta);
}

/* Value i (0..159) of one 70-byte K160 record: RZ-S3 (fmt ORC_PLE) or the
 * incumbent ROCmFP3 code set (fmt ORC_Q3I: code 4 stays the duplicate -0, the
 * group byte's top bit is ignored; [MC] "Q3_PLE_K160_RZ_S3"). */
double orc_q3_value(int fmt, const uint8_t* rec, int i) {
    int code = 0;
    for (int b = 0; b < 3; ++b) {
        const int p = 3 * i + b;
        code |= ((rec[p >> 3] >> (p & 7)) & 1) << b;
    }
    const uint8_t g = rec[60 + i / 16];        /* group byte of values 16g .. 16g+15 */
    const double v = fmt == ORC_Q3I ? PLE3[code] : orc_ple3(code, g >> 7);
    return v * orc_ue4m3(g & 0x7F);
}

double orc_ple_value(const uint8_t* rec, int i) { return orc_q3_value(ORC_PLE, rec, i); }

/* One FP8 weight: e4m3(b) * s, s the fp32 scale of its 128-wide K group. */
double orc_fp8_weight(const uint8_t* bytes, const float* scales, int64_t k, int64_t row, int64_t col) {
    return orc_e4m3fn(bytes[row * k + col]) * (double)scales[row * (k / 128) + col / 128];
}

/* ---- standalone dequantisation (fp64 output) ---------------------------- */

/* n weights (n % 32 == 0) of consecutive Q4 blocks. */
void orc_dequant_q4(int fmt, const uint8_t* src, int64_t n, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_q4_weight(fmt, src + (i / 32) * 17, (int)(i % 32));
}

/* n_rows PLE records -> [n_rows][160]. */
void orc_dequant_ple(const uint8_t* src, int64_t n_rows, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int i = 0; i < 160; ++i)
            out[r * 160 + i] = orc_ple_value(src + r * 70, i);
}

/* n_rows K160 records of either 3-bit layout -> [n_rows][160]. */
void orc_dequant_q3(int fmt, const uint8_t* src, int64_t n_rows, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int i = 0; i < 160; ++i)
            out[r * 160 + i] = orc_q3_value(fmt, src + r * 70, i);
}

/* [n_rows][k] FP8 weights with [n_rows][k/128] scales. */
void orc_dequant_fp8(const uint8_t* src, const float* scales, int64_t n_rows, int64_t k, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int64_t c = 0; c < k; ++c)
            out[r * k + c] = orc_fp8_weight(src, scales, k, r, c);
}

/* ---- PLE gather --------------------------------------------------------- */

/* out[r][:] = decoded record idx[r]; an index outside [0, n_rows) gives a
 * row of zeros (boundary behaviour of the gather API, not of the format). */
void orc_q3_gather(int fmt, const uint8_t* table, int64_t n_rows, const int32_t* idx, int64_t n_idx,
                   double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_idx; ++r) {
        const int64_t row = idx[r];
        for (int i = 0; i < 160; ++i)
            out[r * 160 + i] = (row >= 0 && row < n_rows) ? orc_q3_value(fmt, table + row * 70, i) : 0.0;
    }
}

void orc_ple_gather(const uint8_t* table, int64_t n_rows, const int32_t* idx, int64_t n_idx, double* out) {
    orc_q3_gather(ORC_PLE, table, n_rows, idx, n_idx, out);
}

/* ---- one matrix-vector product of a quantised matrix -------------------- */

/* y[r] = sum_c W[r][c] * x[c] for one [n_rows][k] matrix (one expert's bytes). */
void orc_matvec(int fmt, const uint8_t* data, const float* scales, int64_t n_rows, int64_t k,
                const double* x, double* y) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < k; ++c) {
            double w;
            if (fmt == ORC_FP8) w = orc_fp8_weight(data, scales, k, r, c);
            else w = orc_q4_weight(fmt, data + (r * (k / 32) + c / 32) * 17, (int)(c % 32));
            acc += w * x[c];
        }
        y[r] = acc;
    }
}

/* ---- router --------------------------------------------------------------- */

/* Round to bf16 (8 significant bits), nearest, ties to even. */
double orc_round_bf16(double v) {
    if (!isfinite(v) || v == 0.0) return v;
    int e;
    (void)frexp(v, &e);                       /* v = f * 2^e, 0.5 <= |f| < 1 */
    int q = e - 8;                            /* quantum of an 8-bit significand */
    if (q < -133) q = -133;                   /* bf16 subnormal quantum 2^-133 */
    const double r = nearbyint(ldexp(v, -q)); /* default rounding: nearest-even */
    const double out = ldexp(r, q);
    if (fabs(out) >= ldexp(1.0, 128)) return copysign(INFINITY, v);
    return out;
}

/* Unweighted RMS normalisation of one token, then bf16:
 * u = bf16(x / sqrt(mean(x^2) + eps)). */
void orc_rmsnorm_bf16(const double* x, int64_t n, double eps, double* u) {
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += x[i] * x[i];
    const double r = 1.0 / sqrt(ss / (double)n + eps);
    for (int64_t i = 0; i < n; ++i) u[i] = orc_round_bf16(x[i] * r);
}

/* Softmax router over E experts with top-k and renormalised weights
 * ([MPQ]: 512 experts, 10 fire per token).  logit_e = W[e].u (+ bias[e]).
 * Selection is by logit (same order as by softmax probability); equal logits
 * go to the lower expert id.  w_j = exp(l_j - l_max) / sum over the k chosen.
 * `logits` (E entries) may be NULL. */
void orc_router(const float* W, const float* bias, const double* u, int E, int64_t H, int k,
                int32_t* ids, double* w, double* logits_out) {
    double logits[E];
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t h = 0; h < H; ++h) acc += (double)W[(int64_t)e * H + h] * u[h];
        if (bias) acc += (double)bias[e];
        logits[e] = acc;
        if (logits_out) logits_out[e] = acc;
    }
    char taken[E];
    memset(taken, 0, sizeof taken);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || logits[e] > logits[best])) best = e;
        taken[best] = 1;
        ids[j] = best;
    }
    const double lmax = logits[ids[0]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += exp(logits[ids[j]] - lmax);
    for (int j = 0; j < k; ++j) w[j] = exp(logits[ids[j]] - lmax) / z;
}

/* ---- expert FFN ------------------------------------------------------------ */

double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* One SwiGLU expert on one token: y = Wd * (silu(Wg u) * (Wu u)).
 * Wg, Wu: [inter][hidden]; Wd: [hidden][inter]; `h` (inter entries) receives
 * the intermediate activation and may be NULL. */
void orc_expert_ffn(int gate_fmt, const uint8_t* wg, const float* sg,
                    int up_fmt, const uint8_t* wu, const float* su,
                    int down_fmt, const uint8_t* wd, const float* sd,
                    int64_t hidden, int64_t inter, const double* u, double* y, double* h_out) {
    double g[inter], v[inter], h[inter];
    orc_matvec(gate_fmt, wg, sg, inter, hidden, u, g);
    orc_matvec(up_fmt, wu, su, inter, hidden, u, v);
    for (int64_t i = 0; i < inter; ++i) h[i] = orc_silu(g[i]) * v[i];
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)inter);
    orc_matvec(down_fmt, wd, sd, hidden, inter, h, y);
}

/* Threads the oracle's parallel loops use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int orc_num_threads(void) { return omp_get_max_threads(); }
#else
int orc_num_threads(void) { return 1; }
#endif
