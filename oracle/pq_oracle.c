/*
 * Oracle for the ParetoQ-style per-output-channel weight fake-quantizer.
 *
 * TEST INFRASTRUCTURE ONLY. This file is a plain, slow, single-threaded CPU
 * restatement of what the quantizer computes. It exists so that tests, the
 * smoke check and the CPU baseline leg of the benchmark can compare the CUDA
 * library against something obviously correct. The product path never links,
 * loads or calls it, and it shares no code, header or table with the CUDA
 * sources.
 *
 * Sources (page title and section):
 *  - "ParetoQ, the strongest low-bit QAT I could find" (modelfoundations.com),
 *    section "Finding 3: at low bits, the grid is not a detail": the LSQ
 *    integer grid {-2^(b-1) .. 2^(b-1)-1}*alpha, the SEQ 2-bit levels
 *    {-0.75,-0.25,0.25,0.75}*alpha, the SEQ ternary levels {-2/3,0,2/3}*alpha,
 *    the learnable per-output-channel alpha.
 *  - same page, section "Paper vs. code": the SEQ formula
 *    alpha*(round(Clip(w/alpha)*k/2 - 0.5) + 0.5)/k*2, the per-row scale of
 *    shape (rows, 1), the LSQ alpha gradient with 1/sqrt(n*Qp) scaling, the
 *    STE with clipping-range gate, the clip value 0.99 that removes the
 *    fifth level produced by round-half-even at +1, and the cast of the
 *    quantized weight to the activation dtype with FP32 gradients.
 *  - same page, section "QAT versus PTQ": the STE passes the gradient
 *    straight through inside the clipping range.
 *  - same page, section "The 2-bit recipe, in full": outside the clipping
 *    range the weight gradient is exactly zero while alpha keeps a
 *    boundary-value gradient from the clipped weights.
 *  - "ParetoQ: Improving Scaling Laws in Extremely Low-bit LLM Quantization"
 *    (paperhub.cn rebuttal), section "Regarding more discussion on why SEQ is
 *    better than LSQ": the SEQ code domain {-1.5,-0.5,0.5,1.5}, the ternary
 *    bins [-1.5,-0.5] / [-0.5,0.5] / [0.5,1.5] in the 1.5-scaled domain.
 *  - "Meta's ParetoQ compares five bit widths ..." (llmobile ticker): ternary
 *    weights stored as 2-bit signed integers (the packed code format).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - ternary uses no +-0.5 shift (its printed levels contain zero);
 *  - rounding is round-half-to-even (nearbyintf under FE_TONEAREST);
 *  - clip: +-0.99f for SEQ2, SEQ2_B and ternary; [-1, 1] (mask only) for
 *    binary; the integer bounds for LSQ;
 *  - the STE mask is the closed interval lo <= x <= hi on the unclipped x;
 *  - fp32 operation order: x = w/alpha (IEEE division), xc = clip(x);
 *    SEQ: t = (xc*kh) - 0.5 with two roundings, r = rint(t),
 *    level = (r + 0.5)/kh; ternary: r = rint(xc*1.5), level = r/1.5;
 *    LSQ: r = rint(xc), level = r; then wq32 = level*alpha (one rounding)
 *    and bf16 round-to-nearest-even. The code c is the integer r;
 *  - a zero level keeps the sign of the rounded value (round(-0.3) = -0.0,
 *    so the dequantized weight is -0.0), as the floating-point formula
 *    gives;
 *  - binary: c = (x >= 0) ? +1 : -1 on the unclipped x (sign(+-0) = +1),
 *    level = c;
 *  - d(alpha)_r = grad_scale * sum_j g_j * (level_j - (inside_j ? x_j : 0)),
 *    accumulated in fp64 in column order, stored as fp32;
 *  - packed codes: two's-complement, 2 bits for binary, ternary, SEQ2,
 *    SEQ2_B and LSQ2 (four per byte, column 4j+i in bits [2i+1:2i] of byte
 *    j), 4 bits for LSQ3 and LSQ4 (two per byte, column 2j+i in bits
 *    [4i+3:4i]); rows back to back.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -shared -fPIC
 * (no FMA contraction, so every fp32 step rounds on its own).
 */
#include <fenv.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

/* Quantizer identifiers; the numbering is part of the library's C ABI and
 * is repeated here on purpose (the oracle includes no library header). */
enum {
    PQO_BINARY = 1,
    PQO_TERNARY = 2,
    PQO_SEQ2 = 3,
    PQO_SEQ2_B = 4,
    PQO_LSQ2 = 5,
    PQO_LSQ3 = 6,
    PQO_LSQ4 = 7
};

/* Parameters of one quantizer.
 *   lo, hi : clip range on x = w/alpha (also the STE gate)
 *   kh     : the SEQ "k/2" stretch (1 for LSQ and binary)
 *   shift  : the SEQ half-level shift (0 for ternary, LSQ, binary)
 *   qp     : Q_p of the LSQ gradient scaling rule
 */
typedef struct {
    float lo, hi, kh, shift, qp;
    int is_binary;
    int bits; /* storage width of one packed code: 2, or 4 for LSQ3/LSQ4 */
} pqo_params;

static int pqo_get_params(int q, pqo_params* p) {
    /* 0.99f: the code's clip value 1 - 1e-2 ("Paper vs. code"). */
    const float clip_seq = 0.99f;
    memset(p, 0, sizeof(*p));
    switch (q) {
    case PQO_BINARY:
        p->lo = -1.0f; p->hi = 1.0f; p->kh = 1.0f; p->shift = 0.0f;
        p->qp = 1.0f; p->is_binary = 1; p->bits = 2; return 0;
    case PQO_TERNARY:
        /* scale to [-1.5, 1.5], equal-width bins, no shift */
        p->lo = -clip_seq; p->hi = clip_seq; p->kh = 1.5f; p->shift = 0.0f;
        p->qp = 1.0f; p->bits = 2; return 0;
    case PQO_SEQ2:
        /* k = 2^2 = 4, k/2 = 2: levels (c + 0.5)/2 */
        p->lo = -clip_seq; p->hi = clip_seq; p->kh = 2.0f; p->shift = 0.5f;
        p->qp = 1.5f; p->bits = 2; return 0;
    case PQO_SEQ2_B:
        /* levels {-1.5,-0.5,0.5,1.5}/1.5 */
        p->lo = -clip_seq; p->hi = clip_seq; p->kh = 1.5f; p->shift = 0.5f;
        p->qp = 1.5f; p->bits = 2; return 0;
    case PQO_LSQ2:
    case PQO_LSQ3:
    case PQO_LSQ4: {
        int b = (q == PQO_LSQ2) ? 2 : (q == PQO_LSQ3) ? 3 : 4;
        float half = (float)(1 << (b - 1));
        p->lo = -half; p->hi = half - 1.0f; p->kh = 1.0f; p->shift = 0.0f;
        p->qp = half - 1.0f; p->bits = (b == 2) ? 2 : 4; return 0;
    }
    default:
        return -1;
    }
}

/* bf16 round-to-nearest-even from its definition: add 0x7FFF plus the lowest
 * kept bit, then drop the low 16 bits. NaN inputs are outside the contract. */
uint16_t pqo_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof(u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

float pqo_bf16_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof(f));
    return f;
}

/* One element: code c, level in alpha units, and the fp32 pre-cast
 * dequantized value. clip_hi_override > 0 replaces the symmetric SEQ /
 * ternary clip (used only to reproduce the published equation's literal
 * clip at 1 in a test). Returns -1 on an unknown quantizer. */
int pqo_quantize_scalar(int q, float w, float alpha, float clip_hi_override,
                        int* code, float* level, float* wq32, int* inside,
                        float* x_out) {
    pqo_params p;
    if (pqo_get_params(q, &p)) return -1;
    if (clip_hi_override > 0.0f && !p.is_binary && q != PQO_LSQ2 &&
        q != PQO_LSQ3 && q != PQO_LSQ4) {
        p.lo = -clip_hi_override;
        p.hi = clip_hi_override;
    }
    float x = w / alpha;
    int c;
    float lev;
    if (p.is_binary) {
        c = (x >= 0.0f) ? 1 : -1;
        lev = (float)c;
    } else {
        float xc = x;
        if (xc < p.lo) xc = p.lo;
        if (xc > p.hi) xc = p.hi;
        float r;
        if (p.shift != 0.0f) {
            /* SEQ: round(xc*k/2 - 0.5) + 0.5, divided by k/2 */
            volatile float s = xc * p.kh;   /* first rounding */
            volatile float t = s - p.shift; /* second rounding */
            r = nearbyintf(t);
            volatile float num = r + p.shift;
            lev = num / p.kh;
        } else if (p.kh != 1.0f) {
            /* ternary: round(xc*1.5) divided by 1.5 */
            volatile float s = xc * p.kh;
            r = nearbyintf(s);
            lev = r / p.kh;
        } else {
            /* LSQ: round(xc) on the integer grid */
            r = nearbyintf(xc);
            lev = r;
        }
        /* r is an integer-valued float; a negative argument that rounds to
         * zero gives -0.0, which the level (and the dequantized weight)
         * keeps, as the floating-point formula does. */
        c = (int)r;
    }
    if (code) *code = c;
    if (level) *level = lev;
    if (wq32) {
        volatile float prod = lev * alpha;
        *wq32 = prod;
    }
    if (inside) *inside = (x >= p.lo) && (x <= p.hi);
    if (x_out) *x_out = x;
    return 0;
}

/* Forward: bf16 dequantized weights, int8 codes (nullable) and packed codes
 * (nullable). Packed codes are two's complement, (8/bits) per byte, the
 * first column of a byte in its lowest bits, rows back to back; cols must be
 * a multiple of (8/bits). Returns 0 on success, -1 on a bad argument. */
int pqo_fwd(int q, int64_t rows, int64_t cols, const float* w,
            const float* alpha, uint16_t* wq_bf16, int8_t* codes,
            uint8_t* packed) {
    pqo_params p;
    if (pqo_get_params(q, &p) || rows < 0 || cols < 0) return -1;
    const int64_t per_byte = 8 / p.bits;
    const unsigned mask = (1u << p.bits) - 1u;
    if (packed && cols % per_byte != 0) return -1;
    if (fegetround() != FE_TONEAREST) fesetround(FE_TONEAREST);
    for (int64_t r = 0; r < rows; ++r) {
        const float a = alpha[r];
        for (int64_t j = 0; j < cols; ++j) {
            int c;
            float wq32;
            pqo_quantize_scalar(q, w[r * cols + j], a, 0.0f, &c, NULL, &wq32,
                                NULL, NULL);
            if (wq_bf16) wq_bf16[r * cols + j] = pqo_bf16_rne(wq32);
            if (codes) codes[r * cols + j] = (int8_t)c;
            if (packed) {
                int64_t byte = r * (cols / per_byte) + j / per_byte;
                int slot = (int)(j % per_byte);
                if (slot == 0) packed[byte] = 0;
                packed[byte] |= (uint8_t)(((unsigned)c & mask) << (p.bits * slot));
            }
        }
    }
    return 0;
}

/* Backward: STE-masked fp32 dW and the per-row alpha gradient.
 * row_abs (nullable) receives sum_j |term_j| per row before grad_scale, for
 * the tolerance floor of rows whose sum cancels. */
int pqo_bwd(int q, int64_t rows, int64_t cols, const float* w,
            const float* alpha, const uint16_t* g_bf16, float* dw,
            float* dalpha, float grad_scale, double* row_abs) {
    pqo_params p;
    if (pqo_get_params(q, &p) || rows < 0 || cols < 0) return -1;
    if (fegetround() != FE_TONEAREST) fesetround(FE_TONEAREST);
    for (int64_t r = 0; r < rows; ++r) {
        const float a = alpha[r];
        double acc = 0.0, acc_abs = 0.0;
        for (int64_t j = 0; j < cols; ++j) {
            int inside;
            float lev, x;
            pqo_quantize_scalar(q, w[r * cols + j], a, 0.0f, NULL, &lev, NULL,
                                &inside, &x);
            float g = pqo_bf16_to_float(g_bf16[r * cols + j]);
            if (dw) dw[r * cols + j] = inside ? g : 0.0f;
            double term = (double)g * ((double)lev - (inside ? (double)x : 0.0));
            acc += term;
            acc_abs += fabs(term);
        }
        if (dalpha) dalpha[r] = (float)(acc * (double)grad_scale);
        if (row_abs) row_abs[r] = acc_abs;
    }
    return 0;
}

/* Level of an integer code c in alpha units, by the same formulas as the
 * forward: SEQ (c + shift)/kh, ternary c/1.5, LSQ and binary c. */
static float pqo_level_of_code(const pqo_params* p, int c) {
    if (p->is_binary) return (float)c;
    if (p->shift != 0.0f) {
        volatile float num = (float)c + p->shift;
        return num / p->kh;
    }
    if (p->kh != 1.0f) return (float)c / p->kh;
    return (float)c;
}

/* Dequantize packed codes: read each field (two's complement, `bits` wide,
 * first column in the lowest bits), sign-extend it to the code c, and
 * write bf16_rne(fl(level(c) * alpha)). A zero level gives +0.0: the
 * stored code does not keep the sign of a rounded-to-zero argument.
 * Needs cols % (8/bits) == 0. Returns 0 on success, -1 on a bad argument. */
int pqo_dequant(int q, int64_t rows, int64_t cols, const uint8_t* packed,
                const float* alpha, uint16_t* wq_bf16) {
    pqo_params p;
    if (pqo_get_params(q, &p) || rows < 0 || cols < 0) return -1;
    const int64_t per_byte = 8 / p.bits;
    const unsigned mask = (1u << p.bits) - 1u;
    if (cols % per_byte != 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < cols; ++j) {
            unsigned byte = packed[r * (cols / per_byte) + j / per_byte];
            unsigned f = (byte >> (p.bits * (int)(j % per_byte))) & mask;
            int c = (f & (1u << (p.bits - 1))) ? (int)f - (1 << p.bits) : (int)f;
            volatile float prod = pqo_level_of_code(&p, c) * alpha[r];
            wq_bf16[r * cols + j] = pqo_bf16_rne(prod);
        }
    }
    return 0;
}

/* One AdamW step (decoupled weight decay) on one fp32 parameter, in this
 * fixed fp32 order, each step rounded on its own:
 *   p  = (wd != 0) ? p * decay : p
 *   m  = b1*m + c1*g
 *   v  = b2*v + c2*(g*g)
 *   den = sqrt(v) * inv_sbc2 + eps
 *   p  = p - step * (m / den)
 * with the scalar factors formed once in double from the hyperparameters
 * and rounded to fp32: decay = 1 - lr*wd, b1 = beta1, c1 = 1 - beta1,
 * b2 = beta2, c2 = 1 - beta2, inv_sbc2 = 1/sqrt(1 - beta2^t),
 * step = lr/(1 - beta1^t), eps. */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
    int64_t step;  /* t >= 1 */
} pqo_adamw;

typedef struct {
    float decay, b1, c1, b2, c2, inv_sbc2, step, eps;
    int has_decay;
} pqo_adamw_k;

static pqo_adamw_k pqo_adamw_consts(const pqo_adamw* h) {
    pqo_adamw_k k;
    const double t = (double)h->step;
    k.decay = (float)(1.0 - h->lr * h->weight_decay);
    k.has_decay = h->weight_decay != 0.0;
    k.b1 = (float)h->beta1;
    k.c1 = (float)(1.0 - h->beta1);
    k.b2 = (float)h->beta2;
    k.c2 = (float)(1.0 - h->beta2);
    k.inv_sbc2 = (float)(1.0 / sqrt(1.0 - pow(h->beta2, t)));
    k.step = (float)(h->lr / (1.0 - pow(h->beta1, t)));
    k.eps = (float)h->eps;
    return k;
}

static float pqo_adamw_update(const pqo_adamw_k* k, float p, float g, float* m, float* v) {
    if (k->has_decay) {
        volatile float pd = p * k->decay;
        p = pd;
    }
    volatile float a1 = k->b1 * *m;
    volatile float a2 = k->c1 * g;
    *m = a1 + a2;
    volatile float gg = g * g;
    volatile float b1 = k->b2 * *v;
    volatile float b2 = k->c2 * gg;
    *v = b1 + b2;
    volatile float sq = sqrtf(*v);
    volatile float sc = sq * k->inv_sbc2;
    volatile float den = sc + k->eps;
    volatile float ratio = *m / den;
    volatile float upd = k->step * ratio;
    return p - upd;
}

/* Backward fused with AdamW: computes dW and d(alpha) from the current w
 * and alpha exactly as pqo_bwd, then applies one AdamW step to every
 * weight (gradient dW, states m_w, v_w) and to every row's alpha
 * (gradient: the fp32 d(alpha), states m_a, v_a). w, alpha and the four
 * state arrays are updated in place; dalpha (nullable) receives the fp32
 * d(alpha). hw and ha are the hyperparameters of weights and scales. */
int pqo_bwd_adamw(int q, int64_t rows, int64_t cols, float* w, float* alpha,
                  const uint16_t* g_bf16, float* m_w, float* v_w, float* m_a,
                  float* v_a, float grad_scale, const pqo_adamw* hw,
                  const pqo_adamw* ha, float* dalpha) {
    pqo_params p;
    if (pqo_get_params(q, &p) || rows < 0 || cols < 0 || !hw || !ha) return -1;
    const pqo_adamw_k kw = pqo_adamw_consts(hw), ka = pqo_adamw_consts(ha);
    for (int64_t r = 0; r < rows; ++r) {
        float da;
        if (pqo_bwd(q, 1, cols, w + r * cols, alpha + r, g_bf16 + r * cols, NULL, &da,
                    grad_scale, NULL))
            return -1;
        for (int64_t j = 0; j < cols; ++j) {
            int inside;
            pqo_quantize_scalar(q, w[r * cols + j], alpha[r], 0.0f, NULL, NULL, NULL,
                                &inside, NULL);
            float g = pqo_bf16_to_float(g_bf16[r * cols + j]);
            float dw = inside ? g : 0.0f;
            w[r * cols + j] = pqo_adamw_update(&kw, w[r * cols + j], dw,
                                               &m_w[r * cols + j], &v_w[r * cols + j]);
        }
        alpha[r] = pqo_adamw_update(&ka, alpha[r], da, &m_a[r], &v_a[r]);
        if (dalpha) dalpha[r] = da;
    }
    return 0;
}

/* Backward + AdamW of one row shard whose upstream gradient is the sum of
 * n_src bf16 gradients (one per data-parallel replica, for the same rows):
 * gbar = fl(fl(sum_k g_k) * grad_mult), summed in source order in fp32;
 * then exactly pqo_bwd_adamw's steps with the fp32 gbar in place of g
 * (dW = inside ? gbar : 0; the d(alpha) term is gbar*(level - inside*x)).
 * row_abs (nullable) receives sum_j |term_j| per row before grad_scale, as
 * pqo_bwd gives it, for the tolerance floor of rows whose sum cancels. */
int pqo_reduce_bwd_adamw(int q, int64_t rows, int64_t cols, float* w, float* alpha,
                         int n_src, const uint16_t* const* g_srcs, float grad_mult,
                         float* m_w, float* v_w, float* m_a, float* v_a, float grad_scale,
                         const pqo_adamw* hw, const pqo_adamw* ha, float* dalpha,
                         double* row_abs) {
    pqo_params p;
    if (pqo_get_params(q, &p) || rows < 0 || cols < 0 || n_src < 1 || !g_srcs || !hw || !ha)
        return -1;
    const pqo_adamw_k kw = pqo_adamw_consts(hw), ka = pqo_adamw_consts(ha);
    for (int64_t r = 0; r < rows; ++r) {
        const float a = alpha[r];
        double acc = 0.0, acc_abs = 0.0;
        for (int64_t j = 0; j < cols; ++j) {
            float sum = 0.0f;
            for (int k = 0; k < n_src; ++k) {
                volatile float t = sum + pqo_bf16_to_float(g_srcs[k][r * cols + j]);
                sum = t;
            }
            volatile float gbar = sum * grad_mult;
            int inside;
            float lev, x;
            pqo_quantize_scalar(q, w[r * cols + j], a, 0.0f, NULL, &lev, NULL, &inside, &x);
            const float dw = inside ? gbar : 0.0f;
            const double term = (double)gbar * ((double)lev - (inside ? (double)x : 0.0));
            acc += term;
            acc_abs += fabs(term);
            w[r * cols + j] = pqo_adamw_update(&kw, w[r * cols + j], dw, &m_w[r * cols + j],
                                               &v_w[r * cols + j]);
        }
        const float da = (float)(acc * (double)grad_scale);
        alpha[r] = pqo_adamw_update(&ka, a, da, &m_a[r], &v_a[r]);
        if (dalpha) dalpha[r] = da;
        if (row_abs) row_abs[r] = acc_abs;
    }
    return 0;
}

/* Weight-only low-bit matmul: Y[m][n] = sum_k X[m][k] * level(c[n][k]) *
 * alpha[n], with X bf16 [M, K] row-major, codes packed [N, K*bits/8] as
 * the forward writes them, levels by the forward's formulas taken as exact
 * reals (SEQ2 (2c+1)/4, SEQ2_B (2c+1)/3, ternary 2c/3, LSQ and binary c),
 * evaluated in double. Output fp64 [M, N]. */
int pqo_wq_matmul(int q, int64_t m, int64_t n, int64_t k, const uint16_t* x_bf16,
                  const uint8_t* packed, const float* alpha, double* y) {
    pqo_params p;
    if (pqo_get_params(q, &p) || m < 0 || n < 0 || k < 0) return -1;
    const int64_t per_byte = 8 / p.bits;
    const unsigned mask = (1u << p.bits) - 1u;
    if (k % per_byte != 0) return -1;
    for (int64_t i = 0; i < m; ++i) {
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < k; ++t) {
                unsigned byte = packed[j * (k / per_byte) + t / per_byte];
                unsigned f = (byte >> (p.bits * (int)(t % per_byte))) & mask;
                int c = (f & (1u << (p.bits - 1))) ? (int)f - (1 << p.bits) : (int)f;
                double lev;
                if (p.is_binary || p.kh == 1.0f) lev = (double)c;            /* binary, LSQ */
                else if (p.shift != 0.0f) lev = (2.0 * c + 1.0) / (2.0 * p.kh);  /* SEQ */
                else lev = 2.0 * c / 3.0;                                     /* ternary */
                acc += (double)pqo_bf16_to_float(x_bf16[i * k + t]) * lev;
            }
            y[i * n + j] = acc * (double)alpha[j];
        }
    }
    return 0;
}

/* One AdamW step over n parameters with given gradients (for pinning the
 * update rule against a library optimizer). */
int pqo_adamw_step(int64_t n, float* p, const float* g, float* m, float* v,
                   const pqo_adamw* h) {
    if (n < 0 || !h) return -1;
    const pqo_adamw_k k = pqo_adamw_consts(h);
    for (int64_t i = 0; i < n; ++i) p[i] = pqo_adamw_update(&k, p[i], g[i], &m[i], &v[i]);
    return 0;
}

/* Standalone code export: packed codes only. */
int pqo_pack(int q, int64_t rows, int64_t cols, const float* w,
             const float* alpha, uint8_t* packed) {
    if (!packed) return -1;
    return pqo_fwd(q, rows, cols, w, alpha, NULL, NULL, packed);
}

/* LSQ gradient scaling 1/sqrt(n*Qp) with n = cols (the weights that share
 * one per-row alpha). */
float pqo_default_grad_scale(int q, int64_t cols) {
    pqo_params p;
    if (pqo_get_params(q, &p) || cols <= 0) return 0.0f;
    return (float)(1.0 / sqrt((double)cols * (double)p.qp));
}

int pqo_code_bits(int q) {
    pqo_params p;
    if (pqo_get_params(q, &p)) return -1;
    return p.bits;
}
