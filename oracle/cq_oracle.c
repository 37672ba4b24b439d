/*
 * cq_oracle.c -- plain, slow, obviously correct CPU oracle for group-wise low-bit
 * weight quantization (VBQ per-group bit-widths, CellFill in-cell residuals).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * Sources (the pages are cited by title and section):
 *   [VBQ]  "In-Cell Learning: Language Models That Update Their Own Weights in Sequence
 *          Without Changing the File They Ship" (thelatestinai.com/papers/2608.20873),
 *          abstract: contiguous groups of 64 weights, each group with its own bit-width
 *          from {1,2,4,8}; codes are stored bit-packed at their widths; fused
 *          dequantize-and-multiply kernels for memory-bound decode.
 *   [CF]   "Nothing Changed but the Model: CellFill -- Bounded In-Cell Learning for
 *          Bit-Identical, Revocable Updates to Quantized LLMs", Abstract: 4-bit release
 *          with frozen integer codes and scales; a per-weight residual kept strictly
 *          inside each quantization decision cell; re-quantization returns the release
 *          exactly; removing the residual undoes the update; the weight change is limited.
 *   [SLQ]  same listing page 2 (thelatestinai.com/papers/2512.18934), SLQ abstract:
 *          asymmetric quantization (the reason for the zero point z).
 * The quantizer formula itself is not printed on the pages.  The oracle takes the
 * plainest reading: asymmetric min-max round-to-nearest with an fp16 scale s, a uint8
 * zero z and codes q = clamp(rne(w/s) + z, 0, 2^b - 1), every fp32 operation rounded
 * separately in the order written (see the comments of each function).
 *
 * Build: gcc -std=c99 -O2 -ffp-contract=off -fPIC -shared (no -ffast-math).  On x86-64
 * float arithmetic is SSE scalar binary32 with round-to-nearest-even, and rintf()
 * rounds half to even in the default rounding mode.
 */
#define _POSIX_C_SOURCE 200809L
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* status bits reported by oq_quantize (one word for the whole call) */
#define OQ_ST_NONFINITE 1u /* a group held a NaN or an infinity            */
#define OQ_ST_RANGE 2u     /* the group's scale overflowed fp16            */
#define OQ_ST_BADBITS 4u   /* a group's bit-width was not one of 1,2,4,8   */

#define GROUP 64 /* [VBQ] abstract: contiguous groups of 64 weights */

/* ------------------------------------------------------------------------------
 * Number formats, written from the IEEE-754 definitions.
 * ---------------------------------------------------------------------------- */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* binary32 -> binary16, round to nearest, ties to even.
 * A finite non-zero input is M * 2^(e-23) with a 24-bit integer significand M.
 * The result is m_h * 2^qe, where qe = e-10 in the normal range of binary16 and
 * qe = -24 (the subnormal quantum) below it; m_h = M * 2^(e-23-qe) rounded half-even. */
uint16_t oq_f32_to_f16(float f)
{
    uint32_t x = f2u(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ef = (x >> 23) & 0xFFu, mf = x & 0x7FFFFFu;
    if (ef == 0xFFu) return (uint16_t)(sign | (mf ? 0x7E00u : 0x7C00u));
    if (ef == 0 && mf == 0) return sign;
    uint32_t M = ef ? (mf | 0x800000u) : mf;
    int e = ef ? (int)ef - 127 : -126;
    int normal = e >= -14;
    int qe = normal ? e - 10 : -24;
    int shift = 23 + qe - e; /* >= 13 */
    uint32_t m;
    if (shift >= 32) {
        m = 0; /* M < 2^24 <= half a quantum */
    } else {
        uint32_t rem = M & ((1u << shift) - 1u), half = 1u << (shift - 1);
        m = M >> shift;
        if (rem > half || (rem == half && (m & 1u))) m++;
    }
    if (!normal) return (uint16_t)(sign | m); /* m == 1024 is the smallest normal, bit for bit */
    if (m == 2048u) { m = 1024u; e++; }
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint32_t)(e + 15) << 10) | (m - 1024u));
}

/* binary16 -> binary32 (always exact) */
float oq_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
    if (e == 31) return u2f(sign | 0x7F800000u | (m << 13));
    if (e == 0) {
        float v = ldexpf((float)m, -24); /* m < 1024: exact */
        return sign ? -v : v;
    }
    return u2f(sign | ((e - 15 + 127) << 23) | (m << 13));
}

/* binary32 -> bfloat16, round to nearest even: bfloat16 is the top half of binary32,
 * so rounding drops the low 16 bits with the half-even rule (a carry into the
 * exponent is the correct result, including overflow to infinity). */
uint16_t oq_f32_to_bf16_rn(float f)
{
    uint32_t x = f2u(f);
    if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x7FFFFFu)) return (uint16_t)((x >> 16) | 0x40u);
    uint32_t hi = x >> 16, lo = x & 0xFFFFu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi++;
    return (uint16_t)hi;
}

/* binary32 -> bfloat16, round toward zero: drop the low 16 bits. */
uint16_t oq_f32_to_bf16_rz(float f)
{
    uint32_t x = f2u(f);
    if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x7FFFFFu)) return (uint16_t)((x >> 16) | 0x40u);
    return (uint16_t)(x >> 16);
}

float oq_bf16_to_f32(uint16_t b) { return u2f((uint32_t)b << 16); }

/* array forms of the converters (used by the format tests) */
void oq_f32_to_f16_n(const float *x, uint16_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; i++) y[i] = oq_f32_to_f16(x[i]);
}
void oq_f16_to_f32_n(const uint16_t *x, float *y, int64_t n)
{
    for (int64_t i = 0; i < n; i++) y[i] = oq_f16_to_f32(x[i]);
}
void oq_f32_to_bf16_rn_n(const float *x, uint16_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; i++) y[i] = oq_f32_to_bf16_rn(x[i]);
}
void oq_f32_to_bf16_rz_n(const float *x, uint16_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; i++) y[i] = oq_f32_to_bf16_rz(x[i]);
}

static int valid_bits(int b) { return b == 1 || b == 2 || b == 4 || b == 8; }
static int plane_slot(int b) { return b == 1 ? 0 : b == 2 ? 1 : b == 4 ? 2 : 3; }

/* clamp of an already-rounded integer value v (held exactly as a float) into [0, L]:
 * a float-domain clamp gives the integer clamp's answer without integer overflow,
 * because any v outside [-2^24, 2^24] is far outside [0, L] on the same side. */
static int clamp_code(float v, int L)
{
    if (v < 0.0f) return 0;
    if (v > (float)L) return L;
    return (int)v;
}

/* ------------------------------------------------------------------------------
 * Quantize one group of 64 weights to b bits.
 * Reading (asymmetric min-max RTN, [SLQ] for the asymmetry, [CF] for codes+scales):
 *   wmin, wmax      exact minimum and maximum
 *   s32 = RN32(RN32(wmax - wmin) / L),   L = 2^b - 1
 *   s   = RN_f16(s32); if s < 2^-14 (zero, subnormal) s = 2^-14; s = inf -> RANGE
 *   z   = clamp(rne(RN32(-wmin / s)), 0, L)
 *   q_i = clamp(rne(RN32(w_i / s)) + z, 0, L)
 * A group holding a NaN or infinity, or whose scale overflows, is written as
 * s = +0, z = 0, q = 0 and reported in the status word.
 * ---------------------------------------------------------------------------- */
uint32_t oq_quantize_group(const float *w, int b, uint8_t *q, uint16_t *s_out, uint8_t *z_out)
{
    if (!valid_bits(b)) {
        memset(q, 0, GROUP); *s_out = 0; *z_out = 0;
        return OQ_ST_BADBITS;
    }
    int L = (1 << b) - 1;
    for (int i = 0; i < GROUP; i++) {
        if (!isfinite(w[i])) {
            memset(q, 0, GROUP); *s_out = 0; *z_out = 0;
            return OQ_ST_NONFINITE;
        }
    }
    float wmin = w[0], wmax = w[0];
    for (int i = 1; i < GROUP; i++) {
        if (w[i] < wmin) wmin = w[i];
        if (w[i] > wmax) wmax = w[i];
    }
    float range = wmax - wmin;
    float s32 = range / (float)L;
    uint16_t s16 = oq_f32_to_f16(s32);
    float sf = oq_f16_to_f32(s16);
    if (isinf(sf)) {
        memset(q, 0, GROUP); *s_out = 0; *z_out = 0;
        return OQ_ST_RANGE;
    }
    if (sf < 0x1p-14f) { s16 = 0x0400u; sf = 0x1p-14f; }
    float zq = rintf(-wmin / sf);
    int z = clamp_code(zq, L);
    for (int i = 0; i < GROUP; i++) {
        float t = rintf(w[i] / sf);
        q[i] = (uint8_t)clamp_code(t + (float)z, L);
    }
    *s_out = s16;
    *z_out = (uint8_t)z;
    return 0;
}

/* ------------------------------------------------------------------------------
 * Packed storage ([VBQ]: per-group widths are stored bit-packed).
 * One plane per bit-width b in {1,2,4,8}.  A group of width b occupies 8*b bytes of
 * plane b, starting at byte offset[g]; code j of the group sits in bits
 * [j*b, (j+1)*b) of that little-endian byte string, least significant bit first.
 * offset[g] = 8*b * (number of earlier groups, in row-major group order, with the
 * same width).  A fixed 4-bit release (bits == NULL) uses plane 4 only with
 * offset[g] = 32*g, i.e. plain row-major nibbles, even k in the low nibble.
 * ---------------------------------------------------------------------------- */
int oq_varbits_index(const uint8_t *bits, int64_t G, uint32_t *offset, uint64_t plane_bytes[4])
{
    uint64_t next[4] = {0, 0, 0, 0};
    for (int64_t g = 0; g < G; g++) {
        int b = bits[g];
        if (!valid_bits(b)) return 3;
        int p = plane_slot(b);
        if (next[p] > 0xFFFFFFFFull) return 6; /* byte offsets are 32-bit */
        offset[g] = (uint32_t)next[p];
        next[p] += 8u * (uint64_t)b;
    }
    for (int p = 0; p < 4; p++) plane_bytes[p] = next[p];
    return 0;
}

static uint8_t *group_base(uint8_t *const planes[4], const uint8_t *bits, const uint32_t *offset,
                           int64_t g, int *b_out)
{
    if (!bits) { *b_out = 4; return planes[2] + 32 * g; }
    int b = bits[g];
    *b_out = b;
    return planes[plane_slot(b)] + offset[g];
}

/* codes[G*64] (one code per byte; only the low b bits are stored) -> planes */
int oq_pack(const uint8_t *codes, int64_t G, const uint8_t *bits, const uint32_t *offset,
            uint8_t *plane1, uint8_t *plane2, uint8_t *plane4, uint8_t *plane8)
{
    uint8_t *planes[4] = {plane1, plane2, plane4, plane8};
    for (int64_t g = 0; g < G; g++) {
        int b;
        if (bits && !valid_bits(bits[g])) return 3;
        uint8_t *dst = group_base(planes, bits, offset, g, &b);
        memset(dst, 0, (size_t)(8 * b));
        for (int j = 0; j < GROUP; j++) {
            int code = codes[g * GROUP + j];
            for (int t = 0; t < b; t++) {
                if ((code >> t) & 1) {
                    int pos = j * b + t;
                    dst[pos / 8] |= (uint8_t)(1u << (pos % 8));
                }
            }
        }
    }
    return 0;
}

static int read_code(const uint8_t *src, int b, int j)
{
    int code = 0;
    for (int t = 0; t < b; t++) {
        int pos = j * b + t;
        code |= ((src[pos / 8] >> (pos % 8)) & 1) << t;
    }
    return code;
}

int oq_unpack(const uint8_t *plane1, const uint8_t *plane2, const uint8_t *plane4,
              const uint8_t *plane8, int64_t G, const uint8_t *bits, const uint32_t *offset,
              uint8_t *codes)
{
    uint8_t *planes[4] = {(uint8_t *)plane1, (uint8_t *)plane2, (uint8_t *)plane4, (uint8_t *)plane8};
    for (int64_t g = 0; g < G; g++) {
        int b;
        if (bits && !valid_bits(bits[g])) return 3;
        const uint8_t *src = group_base(planes, bits, offset, g, &b);
        for (int j = 0; j < GROUP; j++) codes[g * GROUP + j] = (uint8_t)read_code(src, b, j);
    }
    return 0;
}

/* ------------------------------------------------------------------------------
 * Projection of the residual into the cell ([CF]: new knowledge lives only in a
 * per-weight residual that may not leave its rounding cell; the dense path clamps
 * into the cells).  Reading: the cell half-width is c = (0.5 - 2^-10) * s for every
 * code (the strict margin 2^-10), c = RN32(0.5-2^-10) * s is exact (9 x 11 bits).
 *   fp32 r:  r <- c if r > c;  -c if r < -c;  r otherwise (a NaN is left as it is)
 *   bf16 r:  the same with c_bf = RZ_bf16(c), so the clamped value is exactly bf16
 *            and never rounds outward.
 * n_clamped counts elements whose bit pattern changed.
 * ---------------------------------------------------------------------------- */
static float cell_halfwidth(uint16_t s16) { return (0.5f - 0x1p-10f) * oq_f16_to_f32(s16); }

static float clamp_into_cell(float r, float c)
{
    if (r > c) return c;
    if (r < -c) return -c;
    return r;
}

int oq_project_f32(float *r, const uint16_t *scale, int64_t n, uint64_t *n_clamped)
{
    uint64_t changed = 0;
    for (int64_t i = 0; i < n; i++) {
        float c = cell_halfwidth(scale[i / GROUP]);
        float v = clamp_into_cell(r[i], c);
        if (f2u(v) != f2u(r[i])) changed++;
        r[i] = v;
    }
    if (n_clamped) *n_clamped = changed;
    return 0;
}

int oq_project_bf16(uint16_t *r, const uint16_t *scale, int64_t n, uint64_t *n_clamped)
{
    uint64_t changed = 0;
    for (int64_t i = 0; i < n; i++) {
        float cb = oq_bf16_to_f32(oq_f32_to_bf16_rz(cell_halfwidth(scale[i / GROUP])));
        float v = clamp_into_cell(oq_bf16_to_f32(r[i]), cb);
        uint16_t vb = (uint16_t)(f2u(v) >> 16); /* v is r or +-cb: exactly bf16 */
        if (vb != r[i]) changed++;
        r[i] = vb;
    }
    if (n_clamped) *n_clamped = changed;
    return 0;
}

/* ------------------------------------------------------------------------------
 * Bounded reparameterization of the residual ([CF] Abstract: CellFill is also offered as a
 * bounded reparameterization, under which staying inside the cell holds by construction
 * instead of being restored by a projection).  The pages do not print the bounded map.
 * Reading: r = RN(c_dt * phi(theta)) with the algebraic sigmoid
 *     phi(theta) = theta / sqrt(1 + theta^2)        (odd, increasing, |phi| < 1, phi(0) = 0)
 * and c_dt the projection's bound for the residual's format (c for fp32, c_bf = RZ_bf16(c)
 * for bf16).  Every step is one IEEE-754 binary32 operation rounded to nearest, in this
 * order, so any IEEE machine reproduces the residual bit for bit:
 *     u = RN(theta * theta);  d = RN(1 + u);  q = RN(sqrt(d));  phi = RN(theta / q)
 * |phi| <= 1 (q >= |theta| in exact arithmetic and RN is monotone), so |r| <= c_dt.
 * |theta| > 2^32 gives phi = +-1 (the value the formula rounds to there; it avoids the
 * overflow of theta^2), and a NaN theta gives r = +0 (its update is revoked): no parameter
 * value, infinities included, can leave the cell.  bf16 r is RN_bf16 of the fp32 product.
 * Backward, straight through the final rounding:
 *     dL/dtheta = RN(RN(dL/dr * c_dt) * phi'),  phi' = (1 + theta^2)^(-3/2) = RN(RN(1 / d) / q)
 * with phi' = 0 for a NaN theta or |theta| > 2^32.
 * ---------------------------------------------------------------------------- */
#define REPARAM_SAT 0x1p32f

float oq_reparam_phi(float theta)
{
    if (theta != theta) return 0.0f;
    if (theta > REPARAM_SAT) return 1.0f;
    if (theta < -REPARAM_SAT) return -1.0f;
    float u = theta * theta;
    float d = 1.0f + u;
    float q = sqrtf(d);
    return theta / q;
}

static float reparam_dphi(float theta)
{
    if (theta != theta || theta > REPARAM_SAT || theta < -REPARAM_SAT) return 0.0f;
    float u = theta * theta;
    float d = 1.0f + u;
    float q = sqrtf(d);
    float inv = 1.0f / d;
    return inv / q;
}

/* the residual's bound in its format (r_dtype 0 = fp32: c, 1 = bf16: c_bf) */
static float reparam_bound(uint16_t s16, int r_dtype)
{
    float c = cell_halfwidth(s16);
    return r_dtype ? oq_bf16_to_f32(oq_f32_to_bf16_rz(c)) : c;
}

int oq_reparam(const float *theta, const uint16_t *scale, int64_t n, int r_dtype, void *r)
{
    for (int64_t i = 0; i < n; i++) {
        float v = reparam_bound(scale[i / GROUP], r_dtype) * oq_reparam_phi(theta[i]);
        if (r_dtype) ((uint16_t *)r)[i] = oq_f32_to_bf16_rn(v);
        else ((float *)r)[i] = v;
    }
    return 0;
}

int oq_reparam_grad(const float *theta, const uint16_t *scale, const float *grad_r, int64_t n, int r_dtype,
                    float *grad_theta)
{
    for (int64_t i = 0; i < n; i++) {
        float gc = grad_r[i] * reparam_bound(scale[i / GROUP], r_dtype);
        grad_theta[i] = gc * reparam_dphi(theta[i]);
    }
    return 0;
}

/* ------------------------------------------------------------------------------
 * Re-quantization check ([CF]: re-quantizing the served weights returns the
 * released artifact bit for bit; dropping the residual revokes exactly).
 * For weight i of group g (code q, scale s, zero z, width b, L = 2^b-1):
 *   k  = q - z
 *   w' = RN32(RN32(s * k) + r_i)           (w' = RN32(s*k) when r is NULL)
 *   t  = RN32(w' / s)
 *   q' = clamp(rne(t) + z, 0, L);  a NaN t counts as a mismatch
 * Outputs: number of i with q' != q, the smallest such i (or -1), and optionally one
 * bit per group of the range, set when the group holds a mismatch.
 * r_dtype: 0 = fp32, 1 = bf16.  first_w must be a multiple of 64.
 * ---------------------------------------------------------------------------- */
static int requant_matches(int q, int z, int L, float sf, const float *r)
{
    float k = (float)(q - z);
    float wp = sf * k;
    if (r) wp = wp + *r;
    float t = wp / sf;
    if (isnan(t)) return 0;
    return clamp_code(rintf(t) + (float)z, L) == q;
}

typedef struct {
    const uint8_t *bits;
    const uint32_t *offset;
    uint8_t *planes[4];
    const uint16_t *scale;
    const uint8_t *zero;
    const void *r;
    int r_dtype;
    int64_t base_w;        /* the call's first weight: group flags are relative to it */
    int64_t lo, hi;        /* this worker's weight range */
    uint32_t *group_flags; /* NULL, or one bit per group of the call's range */
    uint64_t mism;
    int64_t first_bad;
} verify_job;

static void *verify_worker(void *p)
{
    verify_job *J = (verify_job *)p;
    for (int64_t i = J->lo; i < J->hi; i++) {
        int64_t g = i / GROUP;
        int b;
        const uint8_t *src = group_base(J->planes, J->bits, J->offset, g, &b);
        int q = read_code(src, b, (int)(i % GROUP));
        float sf = oq_f16_to_f32(J->scale[g]);
        float rv, *rp = NULL;
        if (J->r) {
            rv = J->r_dtype == 1 ? oq_bf16_to_f32(((const uint16_t *)J->r)[i])
                                 : ((const float *)J->r)[i];
            rp = &rv;
        }
        if (!requant_matches(q, J->zero[g], (1 << b) - 1, sf, rp)) {
            J->mism++;
            if (J->first_bad < 0) J->first_bad = i;
            if (J->group_flags) {
                int64_t gl = g - J->base_w / GROUP;
                J->group_flags[gl / 32] |= 1u << (gl % 32);
            }
        }
    }
    return NULL;
}

#define OQ_MAX_THREADS 256

static int clamp_threads(int n) { return n < 1 ? 1 : n > OQ_MAX_THREADS ? OQ_MAX_THREADS : n; }

int oq_verify(const uint8_t *bits, const uint32_t *offset, const uint8_t *plane1,
              const uint8_t *plane2, const uint8_t *plane4, const uint8_t *plane8,
              const uint16_t *scale, const uint8_t *zero, const void *r, int r_dtype,
              int64_t first_w, int64_t n_w, uint64_t *mismatches, int64_t *first_bad,
              uint32_t *group_flags, int nthreads)
{
    if (first_w < 0 || first_w % GROUP || n_w < 0) return 2;
    int64_t g0 = first_w / GROUP, ngroups = (n_w + GROUP - 1) / GROUP;
    if (bits)
        for (int64_t g = g0; g < g0 + ngroups; g++)
            if (!valid_bits(bits[g])) return 3;
    int64_t words = (ngroups + 31) / 32;
    if (group_flags) memset(group_flags, 0, (size_t)words * 4);
    nthreads = clamp_threads(nthreads);
    /* workers split on 32-group boundaries, so each flag word has one writer */
    int64_t per = (words + nthreads - 1) / nthreads;
    verify_job jobs[OQ_MAX_THREADS];
    pthread_t th[OQ_MAX_THREADS];
    int used = 0;
    for (int t = 0; t < nthreads; t++) {
        int64_t w0 = t * per, w1 = w0 + per;
        if (w1 > words) w1 = words;
        if (w0 >= w1) break;
        verify_job *J = &jobs[used++];
        J->bits = bits; J->offset = offset;
        J->planes[0] = (uint8_t *)plane1; J->planes[1] = (uint8_t *)plane2;
        J->planes[2] = (uint8_t *)plane4; J->planes[3] = (uint8_t *)plane8;
        J->scale = scale; J->zero = zero; J->r = r; J->r_dtype = r_dtype;
        J->base_w = first_w;
        J->lo = first_w + w0 * 32 * GROUP;
        J->hi = first_w + w1 * 32 * GROUP;
        if (J->hi > first_w + n_w) J->hi = first_w + n_w;
        J->group_flags = group_flags; J->mism = 0; J->first_bad = -1;
    }
    if (used == 1) verify_worker(&jobs[0]);
    else {
        for (int t = 0; t < used; t++) pthread_create(&th[t], NULL, verify_worker, &jobs[t]);
        for (int t = 0; t < used; t++) pthread_join(th[t], NULL);
    }
    uint64_t total = 0;
    int64_t fb = -1;
    for (int t = 0; t < used; t++) {
        total += jobs[t].mism;
        if (jobs[t].first_bad >= 0 && (fb < 0 || jobs[t].first_bad < fb)) fb = jobs[t].first_bad;
    }
    *mismatches = total;
    *first_bad = fb;
    return 0;
}

/* ------------------------------------------------------------------------------
 * Whole-matrix quantize: W [rows, cols] row-major, groups of 64 along cols.
 * bits == NULL means every group is 4-bit ([CF]: 4-bit release).
 * ---------------------------------------------------------------------------- */
typedef struct {
    const float *w;
    const uint8_t *bits;
    uint8_t *codes;
    uint16_t *scale;
    uint8_t *zero;
    int64_t g_lo, g_hi;
    uint32_t status;
} quant_job;

static void *quant_worker(void *p)
{
    quant_job *J = (quant_job *)p;
    for (int64_t g = J->g_lo; g < J->g_hi; g++) {
        int b = J->bits ? J->bits[g] : 4;
        J->status |= oq_quantize_group(J->w + g * GROUP, b, J->codes + g * GROUP, J->scale + g,
                                       J->zero + g);
    }
    return NULL;
}

int oq_quantize(const float *w, int64_t rows, int64_t cols, const uint8_t *bits, uint8_t *codes,
                uint16_t *scale, uint8_t *zero, uint32_t *status, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return 2;
    int64_t G = rows * (cols / GROUP);
    nthreads = clamp_threads(nthreads);
    int64_t per = (G + nthreads - 1) / nthreads;
    quant_job jobs[OQ_MAX_THREADS];
    pthread_t th[OQ_MAX_THREADS];
    int used = 0;
    for (int t = 0; t < nthreads; t++) {
        int64_t lo = t * per, hi = lo + per;
        if (hi > G) hi = G;
        if (lo >= hi) break;
        quant_job *J = &jobs[used++];
        J->w = w; J->bits = bits; J->codes = codes; J->scale = scale; J->zero = zero;
        J->g_lo = lo; J->g_hi = hi; J->status = 0;
    }
    if (used == 1) quant_worker(&jobs[0]);
    else if (used > 1) {
        for (int t = 0; t < used; t++) pthread_create(&th[t], NULL, quant_worker, &jobs[t]);
        for (int t = 0; t < used; t++) pthread_join(th[t], NULL);
    }
    uint32_t st = 0;
    for (int t = 0; t < used; t++) st |= jobs[t].status;
    if (status) *status = st;
    return 0;
}

/* ------------------------------------------------------------------------------
 * One stage of Recurrent Residual Quantization.
 * [RRQ] the listing page thelatestinai.com/papers/2512.18934, "Recurrent Residual
 * Quantization" abstract: the weights become a low-bit base plus a sequence of quantized
 * residual corrections; from a 2-bit round-to-nearest base, 2-bit round-to-nearest
 * residuals are added one after another to reach 4, 6 and 8 bits, without calibration.
 * Reading: each stage quantizes the running residual with the group quantizer above at
 * one width b for every group, then the residual becomes what that stage does not
 * represent:
 *     r_i <- RN32(r_i - RN32(s * (q_i - z)))
 * with the stored s, z and q of the stage (s*(q-z) is exact: 11 + 8 significant bits fit
 * in 24).  A group the quantizer flags (s = +0, z = 0, q = 0) keeps its residual.  The
 * first stage is run on the weights themselves, so its codes are the 2-bit base; after
 * stage j the model of the weights is the sum of the stages' s*(q-z).
 * r: rows x cols fp32, replaced in place.  Returns the OR of the groups' status bits.
 * ---------------------------------------------------------------------------- */
uint32_t oq_rrq_stage(float *r, int64_t rows, int64_t cols, int b, uint8_t *codes, uint16_t *scale,
                      uint8_t *zero)
{
    if (rows < 0 || cols < 0 || cols % GROUP) return OQ_ST_BADBITS;
    int64_t G = rows * (cols / GROUP);
    uint32_t st = 0;
    for (int64_t g = 0; g < G; g++) {
        float *rg = r + g * GROUP;
        uint8_t *qg = codes + g * GROUP;
        st |= oq_quantize_group(rg, b, qg, scale + g, zero + g);
        float sf = oq_f16_to_f32(scale[g]);
        float z = (float)zero[g];
        for (int i = 0; i < GROUP; i++) {
            float deq = sf * ((float)qg[i] - z);       /* exact */
            rg[i] = rg[i] - deq;                        /* one rounding */
        }
    }
    return st;
}

/* ------------------------------------------------------------------------------
 * Dequantize-and-multiply reference ([VBQ]: fused dequantize-and-multiply for decode):
 *   y[m, n] = sum_k (s_g * (q[n,k] - z_g) + r[n,k]) * x[m, k]
 * evaluated in binary64: s*(q-z) and every product of binary32/bfloat16 values are
 * exact in binary64, so the only rounding is that of the binary64 sums.
 * x_dtype / r_dtype: 0 = fp32, 1 = bf16.  r may be NULL.  y is [m, rows].
 * ---------------------------------------------------------------------------- */
typedef struct {
    const uint8_t *bits;
    const uint32_t *offset;
    uint8_t *planes[4];
    const uint16_t *scale;
    const uint8_t *zero;
    const void *r;
    int r_dtype;
    const void *x;
    int x_dtype;
    int m;
    int64_t rows, cols;
    int64_t n_lo, n_hi;
    double *y;
} mm_job;

static double load_val(const void *p, int dtype, int64_t i)
{
    return dtype == 1 ? (double)oq_bf16_to_f32(((const uint16_t *)p)[i]) : (double)((const float *)p)[i];
}

static void *mm_worker(void *p)
{
    mm_job *J = (mm_job *)p;
    int64_t gpr = J->cols / GROUP;
    double *wrow = (double *)malloc((size_t)J->cols * sizeof(double));
    if (!wrow) return NULL;
    for (int64_t n = J->n_lo; n < J->n_hi; n++) {
        for (int64_t gk = 0; gk < gpr; gk++) {
            int64_t g = n * gpr + gk;
            int b;
            const uint8_t *src = group_base(J->planes, J->bits, J->offset, g, &b);
            double s = (double)oq_f16_to_f32(J->scale[g]);
            int z = J->zero[g];
            for (int j = 0; j < GROUP; j++) {
                int64_t k = gk * GROUP + j;
                double wv = s * (double)(read_code(src, b, j) - z);
                if (J->r) wv += load_val(J->r, J->r_dtype, n * J->cols + k);
                wrow[k] = wv;
            }
        }
        for (int mi = 0; mi < J->m; mi++) {
            double acc = 0.0;
            for (int64_t k = 0; k < J->cols; k++) acc += wrow[k] * load_val(J->x, J->x_dtype, mi * J->cols + k);
            J->y[mi * J->rows + n] = acc;
        }
    }
    free(wrow);
    return NULL;
}

int oq_dequant_matmul_f64(const uint8_t *bits, const uint32_t *offset, const uint8_t *plane1,
                          const uint8_t *plane2, const uint8_t *plane4, const uint8_t *plane8,
                          const uint16_t *scale, const uint8_t *zero, const void *r, int r_dtype,
                          int64_t rows, int64_t cols, const void *x, int x_dtype, int m,
                          double *y, int nthreads)
{
    if (rows < 0 || cols < 0 || cols % GROUP || m < 1) return 2;
    nthreads = clamp_threads(nthreads);
    int64_t per = (rows + nthreads - 1) / nthreads;
    mm_job jobs[OQ_MAX_THREADS];
    pthread_t th[OQ_MAX_THREADS];
    int used = 0;
    for (int t = 0; t < nthreads; t++) {
        int64_t lo = t * per, hi = lo + per;
        if (hi > rows) hi = rows;
        if (lo >= hi) break;
        mm_job *J = &jobs[used++];
        J->bits = bits; J->offset = offset;
        J->planes[0] = (uint8_t *)plane1; J->planes[1] = (uint8_t *)plane2;
        J->planes[2] = (uint8_t *)plane4; J->planes[3] = (uint8_t *)plane8;
        J->scale = scale; J->zero = zero; J->r = r; J->r_dtype = r_dtype;
        J->x = x; J->x_dtype = x_dtype; J->m = m; J->rows = rows; J->cols = cols;
        J->n_lo = lo; J->n_hi = hi; J->y = y;
    }
    if (used == 1) mm_worker(&jobs[0]);
    else if (used > 1) {
        for (int t = 0; t < used; t++) pthread_create(&th[t], NULL, mm_worker, &jobs[t]);
        for (int t = 0; t < used; t++) pthread_join(th[t], NULL);
    }
    return 0;
}

/* ------------------------------------------------------------------------------
 * ReQuant fixed-grid refinement (page 1, thelatestinai.com/papers/2608.20873, ReQuant
 * abstract: a backpropagation-free stage after any initializer revisits the integer
 * assignments on the fixed grid; an accepted update strictly lowers the mean squared
 * reconstruction error and stays on the grid; several sweeps over a round-to-nearest start).
 * Reading: the error is the layer's output reconstruction error on calibration activations X,
 *     E(q) = sum_n d_n^T H d_n,   d_n = w_n - s (q_n - z),   H = X^T X   (fp64, K x K)
 * (in weight space round-to-nearest is already optimal, so the abstract's gains need the output
 * error); the grid is frozen (s, z unchanged); a candidate update moves one code to a neighbouring
 * level, q +- 1 inside [0, L]. Rows are independent (E separates over rows). For each row, with
 * g = H d kept current: one sweep visits k = 0 .. K-1 in order; with S = s of k's group (exact
 * in fp64), t2 = (S*S)*H_kk, t4 = (2*S)*g_k, the two candidates change E by
 *     up: t2 - t4 (if q_k < L),   down: t2 + t4 (if q_k > 0);
 * the smaller one is taken if it is strictly negative (up on a tie); then q_k moves, and every
 * g_j <- g_j - delta * H_jk with delta = +S or -S. Every operation is one IEEE-754 binary64
 * operation rounded to nearest (no fused multiply-add) and every sum runs in increasing index
 * order, so any implementation that keeps this order reproduces the codes exactly:
 *     d_k = (double)w_k - S*(q_k - z)    (the product exact),
 *     g_j = (...((0 + H_j0 d_0) + H_j1 d_1) ...) + H_j,K-1 d_K-1
 * err_before / err_after (per row, may be NULL): sum_k of d_k * g_k in the same way, with d and
 * g recomputed from scratch; moves (may be NULL): accepted updates per row.
 * ---------------------------------------------------------------------------- */
static void rq_residual(const float *w, const uint16_t *scale, const uint8_t *zero, const uint8_t *q, int64_t K,
                        double *d)
{
    for (int64_t k = 0; k < K; k++) {
        double S = (double)oq_f16_to_f32(scale[k / GROUP]);
        d[k] = (double)w[k] - S * (double)((int)q[k] - (int)zero[k / GROUP]);
    }
}

static void rq_gradient(const double *H, const double *d, int64_t K, double *g)
{
    for (int64_t j = 0; j < K; j++) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; k++) acc = acc + H[j * K + k] * d[k];
        g[j] = acc;
    }
}

static double rq_error(const double *d, const double *g, int64_t K)
{
    double e = 0.0;
    for (int64_t k = 0; k < K; k++) e = e + d[k] * g[k];
    return e;
}

int oq_requant_refine(const float *w, int64_t rows, int64_t cols, const double *H, const uint16_t *scale,
                      const uint8_t *zero, int b, uint8_t *codes, int sweeps, double *err_before,
                      double *err_after, uint64_t *moves)
{
    if (rows < 0 || cols < 0 || cols % GROUP || !valid_bits(b) || sweeps < 0) return 2;
    int64_t K = cols, KG = cols / GROUP;
    int L = (1 << b) - 1;
    double *d = (double *)malloc((size_t)(K ? K : 1) * sizeof(double));
    double *g = (double *)malloc((size_t)(K ? K : 1) * sizeof(double));
    if (!d || !g) { free(d); free(g); return 3; }
    for (int64_t n = 0; n < rows; n++) {
        const float *wn = w + n * K;
        const uint16_t *sn = scale + n * KG;
        const uint8_t *zn = zero + n * KG;
        uint8_t *qn = codes + n * K;
        rq_residual(wn, sn, zn, qn, K, d);
        rq_gradient(H, d, K, g);
        if (err_before) err_before[n] = rq_error(d, g, K);
        uint64_t mv = 0;
        for (int sw = 0; sw < sweeps; sw++) {
            for (int64_t k = 0; k < K; k++) {
                double S = (double)oq_f16_to_f32(sn[k / GROUP]);
                double t2 = (S * S) * H[k * K + k];
                double t4 = (2.0 * S) * g[k];
                double up = t2 - t4, down = t2 + t4;
                int step = 0;
                if (qn[k] < L && up < 0.0) step = 1;
                if (qn[k] > 0 && down < 0.0 && (step == 0 || down < up)) step = -1;
                if (step) {
                    double delta = step > 0 ? S : -S;
                    qn[k] = (uint8_t)(qn[k] + step);
                    for (int64_t j = 0; j < K; j++) g[j] = g[j] - delta * H[j * K + k];
                    mv++;
                }
            }
        }
        if (moves) moves[n] = mv;
        if (err_after) {
            rq_residual(wn, sn, zn, qn, K, d);
            rq_gradient(H, d, K, g);
            err_after[n] = rq_error(d, g, K);
        }
    }
    free(d);
    free(g);
    return 0;
}
