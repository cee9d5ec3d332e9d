// Kernels and C ABI of the ParetoQ-style weight fake-quantizer (sm_100a).
//
// The path is HBM-bound elementwise work (about 10 fp32 operations per 16
// bytes moved), so it uses no tensor cores: 16-byte vector loads and
// stores, one row group per thread group, and a fixed-order per-row
// reduction for the scale gradient.
//
// Layout of the work: a CTA of 256 threads is split into row groups of TPR
// threads (TPR a power of two, 1..256); a row group owns one row at a time
// and walks it in chunks of 8 consecutive weights (two 16-byte loads of W,
// one 16-byte store of bf16 Wq, one 2- or 4-byte store of packed codes).
// The forward may also split a row across CTAs (blockIdx.x); the backward
// keeps a row inside one row group so that the scale gradient is reduced
// in registers, warp shuffles and shared memory, in a fixed order.
//
// Sources: "ParetoQ, the strongest low-bit QAT I could find", sections
// "Finding 3", "Paper vs. code", "QAT versus PTQ", "The 2-bit recipe, in
// full"; "Meta's ParetoQ compares five bit widths ..." (packed 2-bit codes).
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>

#include "pq.h"
#include "pq_quant.cuh"

namespace pq {

constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 8;  // 8 x 256 = 2048 resident threads per SM

// ------------------------------------------------------------ memory helpers
// Number of valid weights in chunk `ch` (8 except in a ragged last chunk).
__device__ __forceinline__ int tail_n(int64_t cols, int64_t ch) {
    const int64_t r = cols - ch * 8;
    return r < 8 ? static_cast<int>(r) : 8;
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8_tail(const float* p, int n, float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (i < n) ? p[i] : 0.0f;
}

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);  // .x -> low half
    return *reinterpret_cast<uint32_t*>(&b);
}

// ------------------------------------------------------------------ forward
// One chunk of 8 weights: bf16 outputs as 4 words, packed codes as one word
// (bits*8 significant bits).
template <int Q, bool WQ, bool PACK>
__device__ __forceinline__ void fwd_chunk(const float (&v)[8], float a,
                                          uint32_t (&h)[4], uint32_t& pk) {
    constexpr int B = Traits<Q>::bits;
    pk = 0;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const Elem e0 = quantize<Q>(v[i], a);
        const Elem e1 = quantize<Q>(v[i + 1], a);
        if constexpr (WQ) {
            h[i / 2] = pack_bf16x2(__fmul_rn(e0.level, a), __fmul_rn(e1.level, a));
        }
        if constexpr (PACK) {
            pk |= code_field<Q>(e0.r) << (B * i);
            pk |= code_field<Q>(e1.r) << (B * (i + 1));
        }
    }
}

template <int Q, bool VEC, bool WQ, bool PACK>
__device__ __forceinline__ void fwd_store(uint16_t* __restrict__ qrow,
                                          uint8_t* __restrict__ prow, int64_t ch,
                                          int n, const uint32_t (&h)[4],
                                          uint32_t pk) {
    constexpr int B = Traits<Q>::bits;
    if constexpr (VEC) {
        if constexpr (WQ)
            __stcs(reinterpret_cast<uint4*>(qrow + ch * 8),
                   make_uint4(h[0], h[1], h[2], h[3]));
        if constexpr (PACK) {
            if constexpr (B == 2)
                __stcs(reinterpret_cast<unsigned short*>(prow + ch * 2),
                       static_cast<unsigned short>(pk));
            else
                __stcs(reinterpret_cast<unsigned int*>(prow + ch * 4), pk);
        }
    } else {
        if constexpr (WQ) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < n) qrow[ch * 8 + i] = static_cast<uint16_t>(h[i / 2] >> (16 * (i & 1)));
        }
        if constexpr (PACK) {
            constexpr int per_byte = 8 / B;
#pragma unroll
            for (int k = 0; k < B; ++k)  // B bytes per chunk of 8 codes
                if (k * per_byte < n) prow[ch * B + k] = static_cast<uint8_t>(pk >> (8 * k));
        }
    }
}

template <int Q, bool VEC, bool WQ, bool PACK>
__global__ void __launch_bounds__(kThreads)
fwd_kernel(const float* __restrict__ w, const float* __restrict__ alpha,
           uint16_t* __restrict__ wq, uint8_t* __restrict__ packed,
           int64_t rows, int64_t cols, int tpr_log2) {
    const int tpr = 1 << tpr_log2;
    const int lane = threadIdx.x & (tpr - 1);
    const int rsub = threadIdx.x >> tpr_log2;
    const int rpb = kThreads >> tpr_log2;
    const int64_t nch = (cols + 7) >> 3;
    const int64_t prow_bytes = cols * Traits<Q>::bits / 8;
    const int64_t cstride = static_cast<int64_t>(gridDim.x) * tpr;

    for (int64_t row = static_cast<int64_t>(blockIdx.y) * rpb + rsub; row < rows;
         row += static_cast<int64_t>(gridDim.y) * rpb) {
        const float a = __ldg(alpha + row);
        const float* wr = w + row * cols;
        uint16_t* qr = WQ ? wq + row * cols : nullptr;
        uint8_t* pr = PACK ? packed + row * prow_bytes : nullptr;
        int64_t ch = static_cast<int64_t>(blockIdx.x) * tpr + lane;
        // two chunks per step: four 16-byte loads in flight per thread
        for (; ch + cstride < nch; ch += 2 * cstride) {
            const int64_t ch1 = ch + cstride;
            float v0[8], v1[8];
            if constexpr (VEC) {
                load8(wr + ch * 8, v0);
                load8(wr + ch1 * 8, v1);
            } else {
                load8_tail(wr + ch * 8, tail_n(cols, ch), v0);
                load8_tail(wr + ch1 * 8, tail_n(cols, ch1), v1);
            }
            uint32_t h0[4], h1[4], p0, p1;
            fwd_chunk<Q, WQ, PACK>(v0, a, h0, p0);
            fwd_chunk<Q, WQ, PACK>(v1, a, h1, p1);
            fwd_store<Q, VEC, WQ, PACK>(qr, pr, ch, tail_n(cols, ch), h0, p0);
            fwd_store<Q, VEC, WQ, PACK>(qr, pr, ch1, tail_n(cols, ch1), h1, p1);
        }
        if (ch < nch) {
            const int n = tail_n(cols, ch);
            float v0[8];
            if constexpr (VEC) load8(wr + ch * 8, v0);
            else load8_tail(wr + ch * 8, n, v0);
            uint32_t h0[4], p0;
            fwd_chunk<Q, WQ, PACK>(v0, a, h0, p0);
            fwd_store<Q, VEC, WQ, PACK>(qr, pr, ch, n, h0, p0);
        }
    }
}

// ----------------------------------------------------------------- backward
// One chunk: dW for 8 weights and their contribution to the row's
// sum_j g_j * (level_j - inside_j * x_j), in fp64 with separate roundings.
template <int Q>
__device__ __forceinline__ double bwd_chunk(const float (&v)[8], const uint32_t (&gw)[4],
                                            float a, float (&d)[8], double acc) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const Elem e = quantize<Q>(v[i], a);
        const uint32_t word = gw[i / 2];
        const float g = (i & 1) ? __uint_as_float(word & 0xFFFF0000u)
                                : __uint_as_float(word << 16);
        d[i] = e.inside ? g : 0.0f;
        const double xm = e.inside ? static_cast<double>(e.x) : 0.0;
        acc = __dadd_rn(acc, __dmul_rn(static_cast<double>(g),
                                       __dsub_rn(static_cast<double>(e.level), xm)));
    }
    return acc;
}

__device__ __forceinline__ void load_g8(const uint16_t* p, uint32_t (&gw)[4]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    gw[0] = u.x; gw[1] = u.y; gw[2] = u.z; gw[3] = u.w;
}

__device__ __forceinline__ void load_g8_tail(const uint16_t* p, int n, uint32_t (&gw)[4]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t lo = (2 * k < n) ? p[2 * k] : 0u;
        const uint32_t hi = (2 * k + 1 < n) ? p[2 * k + 1] : 0u;
        gw[k] = lo | (hi << 16);
    }
}

__device__ __forceinline__ void store8_tail(float* p, int n, const float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < n) p[i] = v[i];
}

template <int Q, bool VEC>
__global__ void __launch_bounds__(kThreads)
bwd_kernel(const float* __restrict__ w, const float* __restrict__ alpha,
           const uint16_t* __restrict__ g, float* __restrict__ dw,
           float* __restrict__ dalpha, float grad_scale, int64_t rows,
           int64_t cols, int tpr_log2) {
    __shared__ double warp_sum[kThreads / 32];
    const int tpr = 1 << tpr_log2;
    const int lane = threadIdx.x & (tpr - 1);
    const int rsub = threadIdx.x >> tpr_log2;
    const int rpb = kThreads >> tpr_log2;
    const int64_t nch = (cols + 7) >> 3;
    const int seg = tpr < 32 ? tpr : 32;

    // block-uniform trip count: every thread reaches every barrier
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * rpb; base < rows;
         base += static_cast<int64_t>(gridDim.x) * rpb) {
        const int64_t row = base + rsub;
        double acc = 0.0;
        if (row < rows) {
            const float a = __ldg(alpha + row);
            const float* wr = w + row * cols;
            const uint16_t* gr = g + row * cols;
            float* dr = dw + row * cols;
            int64_t ch = lane;
            for (; ch + tpr < nch; ch += 2 * tpr) {
                const int64_t ch1 = ch + tpr;
                float v0[8], v1[8], d0[8], d1[8];
                uint32_t g0[4], g1[4];
                if constexpr (VEC) {
                    load8(wr + ch * 8, v0);
                    load_g8(gr + ch * 8, g0);
                    load8(wr + ch1 * 8, v1);
                    load_g8(gr + ch1 * 8, g1);
                } else {
                    const int n0 = tail_n(cols, ch);
                    const int n1 = tail_n(cols, ch1);
                    load8_tail(wr + ch * 8, n0, v0);
                    load_g8_tail(gr + ch * 8, n0, g0);
                    load8_tail(wr + ch1 * 8, n1, v1);
                    load_g8_tail(gr + ch1 * 8, n1, g1);
                }
                acc = bwd_chunk<Q>(v0, g0, a, d0, acc);
                acc = bwd_chunk<Q>(v1, g1, a, d1, acc);
                if constexpr (VEC) {
                    store8(dr + ch * 8, d0);
                    store8(dr + ch1 * 8, d1);
                } else {
                    store8_tail(dr + ch * 8, tail_n(cols, ch), d0);
                    store8_tail(dr + ch1 * 8, tail_n(cols, ch1), d1);
                }
            }
            if (ch < nch) {
                const int n = tail_n(cols, ch);
                float v0[8], d0[8];
                uint32_t g0[4];
                if constexpr (VEC) {
                    load8(wr + ch * 8, v0);
                    load_g8(gr + ch * 8, g0);
                } else {
                    load8_tail(wr + ch * 8, n, v0);
                    load_g8_tail(gr + ch * 8, n, g0);
                }
                acc = bwd_chunk<Q>(v0, g0, a, d0, acc);
                if constexpr (VEC) store8(dr + ch * 8, d0);
                else store8_tail(dr + ch * 8, n, d0);
            }
        }
        // reduce the row group's partial sums in a fixed order
        for (int off = seg >> 1; off > 0; off >>= 1)
            acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off, seg));
        if (tpr > 32) {
            if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = acc;
            __syncthreads();
            if (lane == 0) {
                const int w0 = threadIdx.x >> 5;
                double t = warp_sum[w0];
                for (int k = 1; k < (tpr >> 5); ++k) t = __dadd_rn(t, warp_sum[w0 + k]);
                acc = t;
            }
            __syncthreads();
        }
        if (lane == 0 && row < rows)
            dalpha[row] = static_cast<float>(__dmul_rn(acc, static_cast<double>(grad_scale)));
    }
}

// --------------------------------------------------------------- host side
static thread_local int g_last_cuda_error = 0;

static int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

static inline bool aligned(const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

static inline int ilog2_ceil(int64_t v) {
    int l = 0;
    while ((int64_t{1} << l) < v) ++l;
    return l;
}

// Threads per row: about two chunks of 8 per thread, 1..256.
static inline int choose_tpr_log2(int64_t nch) {
    int l = ilog2_ceil((nch + 1) / 2);
    if (l > 8) l = 8;
    if (l < 0) l = 0;
    return l;
}

static pq_status_t finish_launch() {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        g_last_cuda_error = static_cast<int>(e);
        return PQ_ERR_CUDA;
    }
    return PQ_OK;
}

static int code_bits_of(int q) {
    switch (q) {
        case PQ_BINARY: case PQ_TERNARY: case PQ_SEQ2: case PQ_SEQ2_B: case PQ_LSQ2: return 2;
        case PQ_LSQ3: case PQ_LSQ4: return 4;
        default: return 0;
    }
}

template <int Q, bool VEC>
static void launch_fwd_q(dim3 grid, cudaStream_t s, const float* w, const float* alpha,
                         uint16_t* wq, uint8_t* packed, int64_t rows, int64_t cols, int tl) {
    if (wq && packed)
        fwd_kernel<Q, VEC, true, true><<<grid, kThreads, 0, s>>>(w, alpha, wq, packed, rows, cols, tl);
    else if (wq)
        fwd_kernel<Q, VEC, true, false><<<grid, kThreads, 0, s>>>(w, alpha, wq, packed, rows, cols, tl);
    else
        fwd_kernel<Q, VEC, false, true><<<grid, kThreads, 0, s>>>(w, alpha, wq, packed, rows, cols, tl);
}

template <int Q>
static void launch_fwd_v(bool vec, dim3 grid, cudaStream_t s, const float* w, const float* alpha,
                         uint16_t* wq, uint8_t* packed, int64_t rows, int64_t cols, int tl) {
    if (vec) launch_fwd_q<Q, true>(grid, s, w, alpha, wq, packed, rows, cols, tl);
    else launch_fwd_q<Q, false>(grid, s, w, alpha, wq, packed, rows, cols, tl);
}

static pq_status_t fwd_common(int q, int64_t rows, int64_t cols, const float* w,
                              const float* alpha, uint16_t* wq, uint8_t* packed,
                              void* stream) {
    const int bits = code_bits_of(q);
    if (bits == 0 || rows < 0 || cols < 0) return PQ_ERR_INVALID_ARG;
    if (packed && (cols % (8 / bits)) != 0) return PQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return PQ_OK;
    if (!wq && !packed) return PQ_ERR_INVALID_ARG;
    if (!w || !alpha) return PQ_ERR_INVALID_ARG;

    const bool vec = (cols % 8 == 0) && aligned(w, 16) && (!wq || aligned(wq, 16)) &&
                     (!packed || aligned(packed, bits == 2 ? 2 : 4));
    const int64_t nch = (cols + 7) / 8;
    const int tl = choose_tpr_log2(nch);
    const int64_t tpr = int64_t{1} << tl;
    const int64_t rpb = kThreads / tpr;
    const int64_t row_groups = (rows + rpb - 1) / rpb;
    const int64_t target = static_cast<int64_t>(sm_count()) * kBlocksPerSm;
    int64_t gy = row_groups < 65535 ? row_groups : 65535;
    int64_t gx = 1;
    if (row_groups < target) {  // few rows: split each row across CTAs too
        const int64_t max_gx = (nch + 2 * tpr - 1) / (2 * tpr);
        gx = (target + row_groups - 1) / row_groups;
        if (gx > max_gx) gx = max_gx;
        if (gx < 1) gx = 1;
    }
    const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (q) {
        case PQ_BINARY: launch_fwd_v<PQ_BINARY>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        case PQ_TERNARY: launch_fwd_v<PQ_TERNARY>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        case PQ_SEQ2: launch_fwd_v<PQ_SEQ2>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        case PQ_SEQ2_B: launch_fwd_v<PQ_SEQ2_B>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        case PQ_LSQ2: launch_fwd_v<PQ_LSQ2>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        case PQ_LSQ3: launch_fwd_v<PQ_LSQ3>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        case PQ_LSQ4: launch_fwd_v<PQ_LSQ4>(vec, grid, s, w, alpha, wq, packed, rows, cols, tl); break;
        default: return PQ_ERR_INVALID_ARG;
    }
    return finish_launch();
}

template <int Q>
static void launch_bwd_v(bool vec, unsigned grid, cudaStream_t s, const float* w,
                         const float* alpha, const uint16_t* g, float* dw, float* dalpha,
                         float gs, int64_t rows, int64_t cols, int tl) {
    if (vec)
        bwd_kernel<Q, true><<<grid, kThreads, 0, s>>>(w, alpha, g, dw, dalpha, gs, rows, cols, tl);
    else
        bwd_kernel<Q, false><<<grid, kThreads, 0, s>>>(w, alpha, g, dw, dalpha, gs, rows, cols, tl);
}

}  // namespace pq

using namespace pq;

extern "C" {

pq_status_t pq_fakequant_fwd(pq_quant_t q, int64_t rows, int64_t cols, const float* w,
                             const float* alpha, uint16_t* wq_bf16_out, uint8_t* packed_out,
                             void* stream) {
    if (!wq_bf16_out && rows > 0 && cols > 0) return PQ_ERR_INVALID_ARG;
    return fwd_common(q, rows, cols, w, alpha, wq_bf16_out, packed_out, stream);
}

pq_status_t pq_pack_codes(pq_quant_t q, int64_t rows, int64_t cols, const float* w,
                          const float* alpha, uint8_t* packed_out, void* stream) {
    if (!packed_out && rows > 0 && cols > 0) return PQ_ERR_INVALID_ARG;
    return fwd_common(q, rows, cols, w, alpha, nullptr, packed_out, stream);
}

pq_status_t pq_fakequant_bwd(pq_quant_t q, int64_t rows, int64_t cols, const float* w,
                             const float* alpha, const uint16_t* g_bf16, float* dw_out,
                             float* dalpha_out, float grad_scale, void* stream) {
    if (code_bits_of(q) == 0 || rows < 0 || cols < 0) return PQ_ERR_INVALID_ARG;
    if (rows == 0) return PQ_OK;
    if (!dalpha_out) return PQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cols == 0) {
        if (cudaMemsetAsync(dalpha_out, 0, static_cast<size_t>(rows) * sizeof(float), s) != cudaSuccess)
            return finish_launch();
        return PQ_OK;
    }
    if (!w || !alpha || !g_bf16 || !dw_out) return PQ_ERR_INVALID_ARG;
    const bool vec = (cols % 8 == 0) && aligned(w, 16) && aligned(g_bf16, 16) && aligned(dw_out, 16);
    const int64_t nch = (cols + 7) / 8;
    const int tl = choose_tpr_log2(nch);
    const int64_t rpb = kThreads >> tl;
    const int64_t row_groups = (rows + rpb - 1) / rpb;
    const int64_t cap = static_cast<int64_t>(sm_count()) * kBlocksPerSm * 4;
    const unsigned grid = static_cast<unsigned>(row_groups < cap ? row_groups : cap);
    switch (q) {
        case PQ_BINARY: launch_bwd_v<PQ_BINARY>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        case PQ_TERNARY: launch_bwd_v<PQ_TERNARY>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        case PQ_SEQ2: launch_bwd_v<PQ_SEQ2>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        case PQ_SEQ2_B: launch_bwd_v<PQ_SEQ2_B>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        case PQ_LSQ2: launch_bwd_v<PQ_LSQ2>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        case PQ_LSQ3: launch_bwd_v<PQ_LSQ3>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        case PQ_LSQ4: launch_bwd_v<PQ_LSQ4>(vec, grid, s, w, alpha, g_bf16, dw_out, dalpha_out, grad_scale, rows, cols, tl); break;
        default: return PQ_ERR_INVALID_ARG;
    }
    return finish_launch();
}

int pq_code_bits(pq_quant_t q) { return code_bits_of(q); }

float pq_default_grad_scale(pq_quant_t q, int64_t cols) {
    double qp;
    switch (q) {
        case PQ_BINARY: case PQ_TERNARY: case PQ_LSQ2: qp = 1.0; break;
        case PQ_SEQ2: case PQ_SEQ2_B: qp = 1.5; break;
        case PQ_LSQ3: qp = 3.0; break;
        case PQ_LSQ4: qp = 7.0; break;
        default: return 0.0f;
    }
    if (cols <= 0) return 0.0f;
    return static_cast<float>(1.0 / sqrt(static_cast<double>(cols) * qp));
}

const char* pq_status_string(pq_status_t s) {
    switch (s) {
        case PQ_OK: return "ok";
        case PQ_ERR_INVALID_ARG: return "invalid argument";
        case PQ_ERR_UNSUPPORTED: return "unsupported";
        case PQ_ERR_MISALIGNED: return "misaligned pointer";
        case PQ_ERR_CUDA: return "CUDA runtime error";
        case PQ_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

int pq_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
