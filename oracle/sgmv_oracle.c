/*
 * CPU oracle for SGMV expand-slice.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may load
 * this file's library.  The CUDA library never links, includes or calls it, and
 * it shares no code, header, table or constant with the CUDA library.
 *
 * What it computes ("Implementation: Predibase Lorax SGMV Expand Slice Kernel",
 * sections Description and I/O Contract): for every sequence b with start s_b,
 * length L_b and adapter a = lora_idx[b] (a == -1: no LoRA), and every token
 * m < L_b, with row r = s_b + m,
 *
 *     out[r, off + n] = (add ? out[r, off + n] : 0) + sum_k x[r, k] * B[a][n, k]
 *
 * for n in [0, slice_size); every other element of out keeps its bits.
 *
 * Readings taken where the page is silent (each is listed in the design notes):
 *   - mixed precision: x is first rounded (nearest-even) to the weight dtype;
 *   - products and sums are exact-ish fp64, added in k order 0..K-1 starting
 *     from 0.0; the old output value is added after the sum; ONE rounding
 *     (nearest-even, overflow to infinity) to the output dtype at the end;
 *   - add == 0 overwrites, ignoring the old value (even a NaN);
 *   - an adapter index outside [0, lora_num) leaves the segment untouched;
 *   - a row outside [0, rows of out) or [0, rows of x) is skipped, as is a
 *     segment with a negative start or a non-positive length.
 *
 * The fp16 and bfloat16 conversions below are written from the binary
 * interchange format definitions (IEEE 754-2008 binary16; bfloat16 = the top
 * 16 bits of binary32): sign, biased exponent, fraction, gradual underflow.
 * Parity is pinned by tests/test_oracle_pins.py (brute force, a dense
 * per-adapter matmul, exact integer cases, invariants, the page's worked
 * example, all 65536 bit patterns against the format definition).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F16 = 0, ORC_BF16 = 1, ORC_F32 = 2 };

/* Format parameters: fraction bits f, exponent bits e (bias = 2^(e-1) - 1). */
static int fmt_frac_bits(int dt) { return dt == ORC_F16 ? 10 : 7; }
static int fmt_exp_bits(int dt) { return dt == ORC_F16 ? 5 : 8; }

/* 16-bit pattern -> exact double. */
double orc_decode16(uint16_t bits, int dt)
{
    const int f = fmt_frac_bits(dt), e = fmt_exp_bits(dt);
    const int bias = (1 << (e - 1)) - 1;
    const int sign = (bits >> 15) & 1;
    const int expf = (bits >> f) & ((1 << e) - 1);
    const int frac = bits & ((1 << f) - 1);
    double mag;
    if (expf == (1 << e) - 1) {
        mag = frac ? NAN : INFINITY;
    } else if (expf == 0) {
        /* subnormal: frac * 2^(1 - bias - f) */
        mag = ldexp((double)frac, 1 - bias - f);
    } else {
        mag = ldexp((double)((1 << f) + frac), expf - bias - f);
    }
    return sign ? -mag : mag;
}

/* double -> 16-bit pattern, rounding to nearest, ties to even. */
uint16_t orc_encode16(double v, int dt)
{
    const int f = fmt_frac_bits(dt), e = fmt_exp_bits(dt);
    const int bias = (1 << (e - 1)) - 1;
    const int emin = 1 - bias;         /* exponent of the smallest normal */
    const int emax = bias;             /* exponent of the largest finite */
    const uint16_t sign = signbit(v) ? (uint16_t)0x8000u : (uint16_t)0u;
    const uint16_t inf = (uint16_t)(((1u << e) - 1u) << f);
    if (isnan(v)) return (uint16_t)(sign | inf | (1u << (f - 1)));
    double x = fabs(v);
    if (isinf(x)) return (uint16_t)(sign | inf);
    if (x == 0.0) return sign;

    int ex;
    (void)frexp(x, &ex);               /* x = m * 2^ex, m in [0.5, 1) */
    int E = ex - 1;                    /* floor(log2 x) */
    if (E > emax) return (uint16_t)(sign | inf);
    int qexp = (E < emin ? emin : E) - f;  /* spacing of the grid around x */
    double n = ldexp(x, -qexp);        /* exact: scaling by a power of two */
    double r = floor(n);
    double rem = n - r;
    if (rem > 0.5 || (rem == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;   /* ties to even */
    /* r * 2^qexp is the rounded magnitude; r <= 2^(f+1). */
    if (E < emin) {
        /* subnormal grid; r == 2^f means it rounded up to the smallest normal,
           whose encoding (exponent field 1, fraction 0) is the same integer. */
        return (uint16_t)(sign | (uint16_t)r);
    }
    if (r >= ldexp(1.0, f + 1)) {      /* carried into the next binade */
        E += 1;
        r = ldexp(1.0, f);
        if (E > emax) return (uint16_t)(sign | inf);
    }
    uint32_t expfield = (uint32_t)(E + bias);
    uint32_t frac = (uint32_t)(r - ldexp(1.0, f));
    return (uint16_t)(sign | (expfield << f) | frac);
}

/* Element of a tensor of dtype dt at element index i, as an exact double. */
static double load_elem(const void* p, int dt, int64_t i)
{
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    return orc_decode16(((const uint16_t*)p)[i], dt);
}

/* Round a double to dtype dt and back (the value the dtype can hold). */
static double round_to(double v, int dt)
{
    if (dt == ORC_F32) return (double)(float)v;  /* C's double->float is RN-even */
    return orc_decode16(orc_encode16(v, dt), dt);
}

static void store_elem(void* p, int dt, int64_t i, double v)
{
    if (dt == ORC_F32) ((float*)p)[i] = (float)v;
    else ((uint16_t*)p)[i] = orc_encode16(v, dt);
}

/*
 * The expand-slice operation.  Strides are in elements.
 *   x:  (x_rows, K) of x_dt, element (r, k) at x[r*x_rs + k*x_cs]
 *   w:  (lora_num, N, K) of w_dt, element (a, n, k) at w[a*w_as + n*w_ns + k*w_ks]
 *       (the (lora_num, 1, N, K) layout is the same with its unit dim dropped)
 *   out:(out_rows, H) of out_dt, contiguous row-major, modified in place.
 * If pre != NULL it also receives, for every written element, the fp64 value
 * before the final rounding at pre[r*N + n] (other entries untouched).
 * Returns the number of rows written.
 */
int64_t orc_expand_slice(const void* x, int x_dt, int64_t x_rows, int64_t K, int64_t x_rs, int64_t x_cs,
                         const void* w, int w_dt, int64_t lora_num, int64_t w_as, int64_t w_ns, int64_t w_ks,
                         void* out, int out_dt, int64_t out_rows, int64_t H,
                         const int64_t* seq_start, const int64_t* seq_len, const int64_t* lora_idx,
                         int64_t batches, int64_t slice_offset, int64_t N, int add, double* pre,
                         int nthreads)
{
    int64_t written = 0;
    if (nthreads < 1) nthreads = 1;
    for (int64_t b = 0; b < batches; ++b) {
        const int64_t a = lora_idx[b];
        const int64_t s = seq_start[b];
        const int64_t L = seq_len[b];
        if (a < 0 || a >= lora_num) continue;   /* -1 (and any other invalid id): untouched */
        if (s < 0 || L <= 0) continue;
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads) reduction(+ : written) schedule(static)
#endif
        for (int64_t m = 0; m < L; ++m) {
            const int64_t r = s + m;
            if (r >= out_rows || r >= x_rows) continue;
            /* the row of x cast to the weights' dtype (nearest-even) */
            double* xhat = (double*)malloc((size_t)(K > 0 ? K : 1) * sizeof(double));
            for (int64_t k = 0; k < K; ++k) xhat[k] = round_to(load_elem(x, x_dt, r * x_rs + k * x_cs), w_dt);
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const double wv = load_elem(w, w_dt, a * w_as + n * w_ns + k * w_ks);
                    acc += xhat[k] * wv;
                }
                const int64_t oi = r * H + slice_offset + n;
                const double v = add ? load_elem(out, out_dt, oi) + acc : acc;
                if (pre) pre[r * N + n] = v;
                store_elem(out, out_dt, oi, v);
            }
            free(xhat);
            written += 1;
        }
    }
    return written;
}

/* Vector helpers for the Python side. */
void orc_decode16_array(const uint16_t* bits, double* out, int64_t n, int dt)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_decode16(bits[i], dt);
}

void orc_encode16_array(const double* v, uint16_t* out, int64_t n, int dt)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_encode16(v[i], dt);
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
