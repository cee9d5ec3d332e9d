// Kernels and C ABI of the ParetoQ-style weight fake-quantizer (sm_100a).
//
// The path is HBM-bound elementwise work (about 10 fp32 operations per 16
// bytes moved), so it uses no tensor cores. Design:
//
// * Work unit = (matrix, block of rows[, column segment]). A launch covers
//   a whole batch of matrices (up to 256 descriptors passed as kernel
//   parameters), so a training step's many small and large matrices cost
//   one launch per phase, with no per-matrix ramp-up and tail.
// * A CTA of 256 threads splits into row groups of TPR threads (a power of
//   two, 1..256, chosen per matrix so that each thread owns about sixteen
//   (forward) or eight (backward) chunks of 8 weights of its row). Each
//   thread issues the loads of several chunks (3 in the forward, 2 in the
//   backward) before computing any of them; a chunk's 8 fp32 values move
//   as one 256-bit access, so a warp instruction covers 1024 contiguous
//   bytes.
// * A persistent grid (the occupancy limit; the forward's and backward's
//   registers are capped for 4 CTAs per SM) walks the units in order, so
//   concurrent CTAs stream neighbouring rows. An optional bulk L2 prefetch
//   of each CTA's next unit (cp.async.bulk.prefetch.L2) measured slower and
//   is off.
// * The dequantization of packed codes stages each unit's bf16 output (a
//   block of whole rows, contiguous in memory) in shared memory and writes
//   it with one bulk copy (cp.async.bulk, the TMA engine), double-buffered.
// * The backward reduces the scale gradient per row in a fixed order: fp64
//   partial sums per thread, warp shuffles, then (TPR > 32) one shared-memory
//   slot per warp summed by the group's first thread after a barrier of the
//   group only.
//
// Sources: "ParetoQ, the strongest low-bit QAT I could find", sections
// "Finding 3", "Paper vs. code", "QAT versus PTQ", "The 2-bit recipe, in
// full"; "Meta's ParetoQ compares five bit widths ..." (packed 2-bit codes).
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>

#include "pq.h"
#include "pq_launches.cuh"
#include "pq_quant.cuh"

// Tuning knobs (compile-time; the defaults are the measured choice):
//   PQ_PREFETCH      1: bulk L2 prefetch of each CTA's next unit
//   PQ_CTAS_PER_SM   persistent CTAs per SM (0: the occupancy limit)
//   PQ_CHUNKS_PER_THREAD  target chunks of 8 weights per thread and row
//                    (PQ_FWD_CHUNKS_PER_THREAD: the forward's target)
//   PQ_FWD_UNROLL, PQ_BWD_UNROLL  chunks whose loads a thread issues
//                    before computing any of them (PQ_PACK_UNROLL: the
//                    forward instance that writes packed codes only)
//   PQ_LD_HINT, PQ_ST_HINT  cache hints of the streaming loads and stores
//                    (loads: 0 evict-first, 1 read-only path, 2 default,
//                    3 evict-first with a 256-byte L2 prefetch, 4 read-only
//                    without L1 allocation with a 256-byte L2 prefetch)
//   PQ_BWD_MIN_CTAS  resident CTAs per SM the backward's registers must allow
//   PQ_FWD_MIN_CTAS  the same for the forward (PQ_PACK_MIN_CTAS: its
//                    packed-codes-only instance; PQ_RED_MIN_CTAS: the
//                    sharded reduce + backward + AdamW)
//   PQ_DEQ_BULK      1: the dequantization stages each unit's bf16 output in
//                    shared memory and writes it with one bulk copy
//   PQ_DEQ_BUF_KB    size of one such staging buffer (two per CTA)
#ifndef PQ_PREFETCH
#define PQ_PREFETCH 0
#endif
#ifndef PQ_CTAS_PER_SM
#define PQ_CTAS_PER_SM 0
#endif
#ifndef PQ_CHUNKS_PER_THREAD
#define PQ_CHUNKS_PER_THREAD 8
#endif
#ifndef PQ_FWD_CHUNKS_PER_THREAD
#define PQ_FWD_CHUNKS_PER_THREAD 16
#endif
#ifndef PQ_FWD_UNROLL
#define PQ_FWD_UNROLL 3
#endif
#ifndef PQ_PACK_UNROLL
#define PQ_PACK_UNROLL 4
#endif
#ifndef PQ_BWD_UNROLL
#define PQ_BWD_UNROLL 2
#endif
#ifndef PQ_LD_HINT
#define PQ_LD_HINT 0
#endif
#ifndef PQ_BWD_MIN_CTAS
#define PQ_BWD_MIN_CTAS 4
#endif
#ifndef PQ_ST_HINT
#define PQ_ST_HINT 0
#endif
#ifndef PQ_FWD_MIN_CTAS
#define PQ_FWD_MIN_CTAS 4
#endif
#ifndef PQ_DEQ_BULK
#define PQ_DEQ_BULK 1
#endif
#ifndef PQ_DEQ_BUF_KB
#define PQ_DEQ_BUF_KB 32
#endif
#ifndef PQ_PACK_MIN_CTAS
#define PQ_PACK_MIN_CTAS 3
#endif
#ifndef PQ_RED_MIN_CTAS
#define PQ_RED_MIN_CTAS 3
#endif

std::atomic<int64_t> pqc::launches{0};

namespace pq {

constexpr int kThreads = 256;
#ifndef PQ_MAX_BATCH
#define PQ_MAX_BATCH 256
#endif
constexpr int kMaxBatch = PQ_MAX_BATCH;  // descriptors per launch

// ------------------------------------------------------------ memory helpers
// Number of valid weights in chunk `ch` (8 except in a ragged last chunk).
__device__ __forceinline__ int tail_n(int64_t cols, int64_t ch) {
    const int64_t r = cols - ch * 8;
    return r < 8 ? static_cast<int>(r) : 8;
}

// Streaming load/store flavours (PQ_LD_HINT: 0 evict-first, 1 read-only
// path, 2 default; PQ_ST_HINT: 0 evict-first, 1 default).
template <typename T>
__device__ __forceinline__ T ld_stream(const T* p) {
#if PQ_LD_HINT == 0
    return __ldcs(p);
#elif PQ_LD_HINT == 1
    return __ldg(p);
#else
    return *p;
#endif
}
template <typename T>
__device__ __forceinline__ void st_stream(T* p, T v) {
#if PQ_ST_HINT == 0
    __stcs(p, v);
#else
    *p = v;
#endif
}

// Eight consecutive fp32 values (32-byte aligned) as one 256-bit access, so
// a warp's access covers 1024 contiguous bytes (two 16-byte accesses per
// lane would each cover only half of every 32-byte sector).
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
#if PQ_LD_HINT == 0
    asm("ld.global.cs.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "l"(p));
#elif PQ_LD_HINT == 3
    asm("ld.global.cs.L2::256B.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "l"(p));
#elif PQ_LD_HINT == 4
    asm("ld.global.nc.L1::no_allocate.L2::256B.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "l"(p));
#else
    const float4 a = ld_stream(reinterpret_cast<const float4*>(p));
    const float4 b = ld_stream(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
#endif
}

__device__ __forceinline__ void load8_tail(const float* p, int n, float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (i < n) ? p[i] : 0.0f;
}

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
#if PQ_ST_HINT == 0
    asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0]), "f"(v[1]),
                 "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
#else
    st_stream(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    st_stream(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
#endif
}

__device__ __forceinline__ void store8_tail(float* p, int n, const float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < n) p[i] = v[i];
}

__device__ __forceinline__ void load_g8(const uint16_t* p, uint32_t (&gw)[4]) {
    const uint4 u = ld_stream(reinterpret_cast<const uint4*>(p));
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);  // .x -> low half
    return *reinterpret_cast<uint32_t*>(&b);
}

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, int64_t bytes) {
    const char* c = static_cast<const char*>(p);
    while (bytes > 0) {
        const uint32_t n = bytes > (1 << 20) ? (1u << 20) : static_cast<uint32_t>(bytes);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(c), "r"(n) : "memory");
        c += n;
        bytes -= n;
    }
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Barrier over the `count` threads of one row group (ids 1..8; id 0 is
// __syncthreads). All threads of the group reach it equally often.
__device__ __forceinline__ void group_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------------- chunk math
// Forward of one chunk of 8 weights: bf16 outputs as 4 words, packed codes
// as one word (bits*8 significant bits).
template <int Q, bool WQ, bool PACK>
__device__ __forceinline__ void fwd_chunk(const float (&v)[8], const RowScale& s,
                                          uint32_t (&h)[4], uint32_t& pk) {
    constexpr int B = Traits<Q>::bits;
    float x[8];
    divide8(v, s, x);
    pk = 0;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const Elem e0 = quantize_x<Q>(x[i]);
        const Elem e1 = quantize_x<Q>(x[i + 1]);
        if constexpr (WQ) {
            h[i / 2] = pack_bf16x2(__fmul_rn(e0.level, s.a), __fmul_rn(e1.level, s.a));
        }
        if constexpr (PACK) {
            pk |= code_field<Q>(e0) << (B * i);
            pk |= code_field<Q>(e1) << (B * (i + 1));
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
            st_stream(reinterpret_cast<uint4*>(qrow + ch * 8),
                      make_uint4(h[0], h[1], h[2], h[3]));
        if constexpr (PACK) {
            if constexpr (B == 2)
                st_stream(reinterpret_cast<unsigned short*>(prow + ch * 2),
                          static_cast<unsigned short>(pk));
            else
                st_stream(reinterpret_cast<unsigned int*>(prow + ch * 4), pk);
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

// Backward of one chunk: dW for 8 weights and their contribution to the
// row's sum_j g_j * (level_j - inside_j * x_j), accumulated in fp64.
template <int Q>
__device__ __forceinline__ double bwd_chunk(const float (&v)[8], const uint32_t (&gw)[4],
                                            const RowScale& s, float (&d)[8], double acc) {
    float x[8];
    divide8(v, s, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const Elem e = quantize_x<Q>(x[i]);
        const uint32_t word = gw[i / 2];
        const float g = (i & 1) ? __uint_as_float(word & 0xFFFF0000u)
                                : __uint_as_float(word << 16);
        d[i] = e.inside ? g : 0.0f;
        const float xm = e.inside ? x[i] : 0.0f;
        // level - xm is exact in fp64; the product and the sum round once
        acc = __fma_rn(static_cast<double>(g),
                       __dsub_rn(static_cast<double>(e.level), static_cast<double>(xm)), acc);
    }
    return acc;
}

// Backward of one chunk with an fp32 upstream gradient (already reduced).
template <int Q>
__device__ __forceinline__ double bwd_chunk_f32(const float (&v)[8], const float (&g)[8],
                                                const RowScale& s, float (&d)[8], double acc) {
    float x[8];
    divide8(v, s, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const Elem e = quantize_x<Q>(x[i]);
        d[i] = e.inside ? g[i] : 0.0f;
        const float xm = e.inside ? x[i] : 0.0f;
        acc = __fma_rn(static_cast<double>(g[i]),
                       __dsub_rn(static_cast<double>(e.level), static_cast<double>(xm)), acc);
    }
    return acc;
}

// ------------------------------------------------------------ batches
// Device-side descriptor of one matrix of a batch (kernel parameter space).
struct MatDesc {
    const float* w;
    const float* alpha;
    uint16_t* wq;          // forward bf16 output (nullable)
    uint8_t* packed;       // forward packed codes (nullable)
    const uint16_t* g;     // backward upstream gradient
    float* dw;             // backward dW
    float* dalpha;         // backward d(alpha)
    int64_t rows;
    int64_t cols;
    int64_t unit_begin;    // first unit of this matrix in the batch
    float grad_scale;
    int32_t tpr_log2;      // threads per row = 1 << tpr_log2
    int32_t col_splits;    // forward: column segments per row block
    int32_t pad_;
};

// Descriptors of one launch, passed as the kernel's parameter block. A
// launch of at most kSmallBatch matrices uses the small instantiation: its
// parameter block is 24 KB smaller, which shortens the launch (about 2 us
// measured on one small matrix).
constexpr int kSmallBatch = 8;

template <typename D, int CAP = kMaxBatch>
struct BatchT {
    int32_t n;
    int32_t pad_;
    int64_t total_units;
    D m[CAP];
};
using Batch = BatchT<MatDesc>;
template <int CAP>
using MatBatch = BatchT<MatDesc, CAP>;

// Moves `mi` forward to the matrix that owns unit u (units increase).
template <typename D, int CAP>
__device__ __forceinline__ int find_matrix(const BatchT<D, CAP>& p, int mi, int64_t u) {
    while (mi + 1 < p.n && p.m[mi + 1].unit_begin <= u) ++mi;
    return mi;
}

// Bulk L2 prefetch of the inputs of unit u (vector layout only).
template <bool BWD, int CAP>
__device__ __forceinline__ void prefetch_unit(const MatBatch<CAP>& p, int mi, int64_t u) {
    if (u >= p.total_units) return;
    mi = find_matrix(p, mi, u);
    const MatDesc& m = p.m[mi];
    if (m.col_splits != 1) return;
    const int64_t rpb = kThreads >> m.tpr_log2;
    const int64_t r0 = (u - m.unit_begin) * rpb;
    const int64_t nr = (m.rows - r0) < rpb ? (m.rows - r0) : rpb;
    prefetch_l2(m.w + r0 * m.cols, nr * m.cols * 4);
    if constexpr (BWD) prefetch_l2(m.g + r0 * m.cols, nr * m.cols * 2);
}

// ------------------------------------------------------------------ forward
template <int Q, bool VEC, bool WQ, bool PACK, int CAP>
__global__ void __launch_bounds__(kThreads, WQ ? PQ_FWD_MIN_CTAS : PQ_PACK_MIN_CTAS)
fwd_units_kernel(const __grid_constant__ MatBatch<CAP> p) {
    int mi = 0;
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x) {
        mi = find_matrix(p, mi, u);
        const MatDesc& m = p.m[mi];
        if (VEC && PQ_PREFETCH && threadIdx.x == 0) prefetch_unit<false, CAP>(p, mi, u + gridDim.x);
        const int tl = m.tpr_log2;
        const int tpr = 1 << tl;
        const int lane = threadIdx.x & (tpr - 1);
        const int rpb = kThreads >> tl;
        const int64_t lu = u - m.unit_begin;
        const int64_t row = (lu / m.col_splits) * rpb + (threadIdx.x >> tl);
        if (row >= m.rows) continue;
        const int64_t nch = (m.cols + 7) >> 3;
        // chunk range of this unit's column segment
        const int64_t seg = (nch + m.col_splits - 1) / m.col_splits;
        const int64_t c_begin = (lu % m.col_splits) * seg;
        const int64_t c_end = (c_begin + seg) < nch ? (c_begin + seg) : nch;
        const RowScale a = row_scale(__ldg(m.alpha + row));
        const float* wr = m.w + row * m.cols;
        uint16_t* qr = WQ ? m.wq + row * m.cols : nullptr;
        uint8_t* pr = PACK ? m.packed + row * (m.cols * Traits<Q>::bits / 8) : nullptr;
        // chunks in flight: the packed-codes-only instance keeps no bf16
        // outputs live, so it can hold more; element path: fewer registers
        constexpr int U = VEC ? (WQ ? PQ_FWD_UNROLL : PQ_PACK_UNROLL) : 2;
        for (int64_t ch = c_begin + lane; ch < c_end; ch += U * tpr) {
            float v[U][8];
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int64_t c = ch + k * tpr;
                if (c < c_end) {
                    if constexpr (VEC) load8(wr + c * 8, v[k]);
                    else load8_tail(wr + c * 8, tail_n(m.cols, c), v[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int64_t c = ch + k * tpr;
                if (c < c_end) {
                    uint32_t h[4], pk;
                    fwd_chunk<Q, WQ, PACK>(v[k], a, h, pk);
                    fwd_store<Q, VEC, WQ, PACK>(qr, pr, c, tail_n(m.cols, c), h, pk);
                }
            }
        }
    }
}

// ----------------------------------------------------------------- backward
template <int Q, bool VEC, int CAP>
__global__ void __launch_bounds__(kThreads, PQ_BWD_MIN_CTAS)
bwd_units_kernel(const __grid_constant__ MatBatch<CAP> p) {
    __shared__ double warp_sum[2][kThreads / 32];
    int mi = 0, prev_mi = 0, parity = 0;
    // block-uniform trip count: every thread reaches every barrier
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x, parity ^= 1) {
        mi = find_matrix(p, mi, u);
        // a new matrix may regroup the threads: let every group finish
        // reading the previous slots first
        if (mi != prev_mi) __syncthreads();
        prev_mi = mi;
        const MatDesc& m = p.m[mi];
        if (VEC && PQ_PREFETCH && threadIdx.x == 0) prefetch_unit<true, CAP>(p, mi, u + gridDim.x);
        const int tl = m.tpr_log2;
        const int tpr = 1 << tl;
        const int lane = threadIdx.x & (tpr - 1);
        const int rsub = threadIdx.x >> tl;
        const int rpb = kThreads >> tl;
        const int64_t row = (u - m.unit_begin) * rpb + rsub;
        const int64_t nch = (m.cols + 7) >> 3;
        double acc = 0.0;
        if (row < m.rows) {
            const RowScale a = row_scale(__ldg(m.alpha + row));
            const float* wr = m.w + row * m.cols;
            const uint16_t* gr = m.g + row * m.cols;
            float* dr = m.dw + row * m.cols;
            constexpr int U = PQ_BWD_UNROLL;
            for (int64_t ch = lane; ch < nch; ch += U * tpr) {
                float v[U][8];
                uint32_t gw[U][4];
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int64_t c = ch + k * tpr;
                    if (c < nch) {
                        if constexpr (VEC) {
                            load8(wr + c * 8, v[k]);
                            load_g8(gr + c * 8, gw[k]);
                        } else {
                            const int n = tail_n(m.cols, c);
                            load8_tail(wr + c * 8, n, v[k]);
                            load_g8_tail(gr + c * 8, n, gw[k]);
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int64_t c = ch + k * tpr;
                    if (c < nch) {
                        float d[8];
                        acc = bwd_chunk<Q>(v[k], gw[k], a, d, acc);
                        if constexpr (VEC) store8(dr + c * 8, d);
                        else store8_tail(dr + c * 8, tail_n(m.cols, c), d);
                    }
                }
            }
        }
        // reduce the row group's partial sums in a fixed order
        const int seg = tpr < 32 ? tpr : 32;
        for (int off = seg >> 1; off > 0; off >>= 1)
            acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off, seg));
        if (tpr > 32) {
            if ((threadIdx.x & 31) == 0) warp_sum[parity][threadIdx.x >> 5] = acc;
            group_barrier(1 + rsub, tpr);
            if (lane == 0) {
                const int w0 = threadIdx.x >> 5;
                double t = warp_sum[parity][w0];
                for (int k = 1; k < (tpr >> 5); ++k) t = __dadd_rn(t, warp_sum[parity][w0 + k]);
                acc = t;
            }
        }
        if (lane == 0 && row < m.rows)
            m.dalpha[row] = static_cast<float>(__dmul_rn(acc, static_cast<double>(m.grad_scale)));
    }
}

// ------------------------------------------------------- scaled weights
// x = RN(w / alpha_row) with the division routine of the quantizer kernels.
__global__ void __launch_bounds__(kThreads)
scaled_weights_kernel(const float* __restrict__ w, const float* __restrict__ alpha,
                      float* __restrict__ x, int64_t rows, int64_t cols) {
    const int64_t nch = (cols + 7) >> 3;
    for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const RowScale s = row_scale(__ldg(alpha + row));
        for (int64_t ch = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; ch < nch;
             ch += static_cast<int64_t>(gridDim.x) * kThreads) {
            const int n = tail_n(cols, ch);
            float v[8], q[8];
            load8_tail(w + row * cols + ch * 8, n, v);
            divide8(v, s, q);
            store8_tail(x + row * cols + ch * 8, n, q);
        }
    }
}

// ----------------------------------------------------------- dequantize
// Packed codes -> bf16(fl(level * alpha)), over a batch of matrices in the
// same (matrix, row block) units as the forward. In a batch descriptor,
// `packed` is the input (codes a forward wrote) and `wq` the output.
//
// Vector layout (cols % 8 == 0, aligned): lane l of a row group decodes
// chunks of 8 codes l, l + TPR, ..., four loads in flight, so each warp
// store writes 512 contiguous bytes. 2-bit codes: the row's four possible
// outputs form a table held byte-planar in two registers (lo = low bytes of
// entries 0..3, hi = high bytes), so one byte permute (PRMT) decodes two
// weights; its selectors come from spreading a byte's four 2-bit fields to
// byte positions with two overlap-free multiplies (even fields by 1 + 2^12,
// odd ones by 2^6 + 2^18). 4-bit codes and the element path decode each
// field arithmetically.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    return __byte_perm(a, b, sel);
}

// Fields of byte b (4 codes of 2 bits) moved to bits 0, 8, 16, 24.
__device__ __forceinline__ uint32_t spread2(uint32_t b) {
    return ((b & 0x33u) * 0x1001u | (b & 0xCCu) * 0x40040u) & 0x03030303u;
}

// Eight codes of one chunk (2-bit: 16 bits of pk; 4-bit: 32 bits) as eight
// bf16 outputs. 2-bit: byte permutes of the row's table (lo, hi);
// 4-bit: arithmetic decode and one fp32 multiply each.
template <int Q>
__device__ __forceinline__ uint4 dequant_chunk(uint32_t pk, uint32_t lo, uint32_t hi, float a) {
    constexpr int B = Traits<Q>::bits;
    constexpr uint32_t mask = (1u << B) - 1u;
    uint32_t o[4];
    if constexpr (B == 2) {
        const uint32_t t0 = spread2(pk & 0xFFu);
        const uint32_t t1 = spread2(pk >> 8);
        o[0] = prmt(lo, hi, t0 * 0x11u + 0x4040u);
        o[1] = prmt(lo, hi, (t0 >> 16) * 0x11u + 0x4040u);
        o[2] = prmt(lo, hi, t1 * 0x11u + 0x4040u);
        o[3] = prmt(lo, hi, (t1 >> 16) * 0x11u + 0x4040u);
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = pack_bf16x2(__fmul_rn(level_of_field<Q>((pk >> (8 * j)) & mask), a),
                               __fmul_rn(level_of_field<Q>((pk >> (8 * j + 4)) & mask), a));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The row's four 2-bit outputs as a byte-planar table (lo = low bytes of
// entries 0..3, hi = high bytes) for dequant_chunk.
template <int Q>
__device__ __forceinline__ void dequant_table(float a, uint32_t& lo, uint32_t& hi) {
    const uint32_t e01 = pack_bf16x2(__fmul_rn(level_of_field<Q>(0), a),
                                     __fmul_rn(level_of_field<Q>(1), a));
    const uint32_t e23 = pack_bf16x2(__fmul_rn(level_of_field<Q>(2), a),
                                     __fmul_rn(level_of_field<Q>(3), a));
    lo = prmt(e01, e23, 0x6420);
    hi = prmt(e01, e23, 0x7531);
}

// ---------------------------------------------- bulk (TMA engine) stores
constexpr int kDeqBuf = PQ_DEQ_BUF_KB * 1024;        // bytes of one staging buffer
constexpr int kDeqChunks = kDeqBuf / (kThreads * 16);  // chunks per thread that fill it

__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(ssrc), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the bulk stores of all but the newest group have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Vector-layout dequantization with staged output: a unit (a block of whole
// rows, at most kDeqBuf bytes of bf16 output, contiguous in memory) is
// decoded into one of two shared-memory buffers, then written by a single
// bulk copy that thread 0 issues; the other buffer is filled meanwhile.
// Thread 0 waits for a buffer's previous copy to finish reading before the
// CTA refills it. Every thread reaches both barriers of every unit.
template <int Q, int CAP>
__global__ void __launch_bounds__(kThreads)
dequant_bulk_kernel(const __grid_constant__ MatBatch<CAP> p) {
    constexpr int B = Traits<Q>::bits;
    extern __shared__ __align__(128) uint8_t sbuf[];
    int mi = 0;
    uint32_t it = 0;
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x, ++it) {
        mi = find_matrix(p, mi, u);
        const MatDesc& m = p.m[mi];
        const int tl = m.tpr_log2;
        const int tpr = 1 << tl;
        const int lane = threadIdx.x & (tpr - 1);
        const int rsub = threadIdx.x >> tl;
        const int rpb = kThreads >> tl;
        const int64_t row0 = (u - m.unit_begin) * rpb;
        const int64_t row = row0 + rsub;
        const int64_t nrows = (m.rows - row0) < rpb ? (m.rows - row0) : rpb;
        const int64_t nch = m.cols >> 3;
        const bool live = row < m.rows;
        // this thread's codes (at most kDeqChunks chunks of its row)
        uint32_t pk[kDeqChunks];
        float a = 0.0f;
        if (live) {
            a = __ldg(m.alpha + row);
            const uint8_t* src = m.packed + row * (m.cols * B / 8);
#pragma unroll
            for (int k = 0; k < kDeqChunks; ++k) {
                const int64_t c = lane + static_cast<int64_t>(k) * tpr;
                if (c < nch) {
                    if constexpr (B == 2)
                        pk[k] = ld_stream(reinterpret_cast<const unsigned short*>(src + c * 2));
                    else
                        pk[k] = ld_stream(reinterpret_cast<const unsigned int*>(src + c * 4));
                }
            }
        }
        uint8_t* buf = sbuf + (it & 1u) * kDeqBuf;
        if (threadIdx.x == 0) bulk_wait_read_all_but_one();
        __syncthreads();
        if (live) {
            uint32_t lo = 0, hi = 0;
            if constexpr (B == 2) dequant_table<Q>(a, lo, hi);
            const uint32_t rbase = smem_addr(buf) + static_cast<uint32_t>(rsub * m.cols * 2);
#pragma unroll
            for (int k = 0; k < kDeqChunks; ++k) {
                const int64_t c = lane + static_cast<int64_t>(k) * tpr;
                if (c < nch) {
                    const uint4 o = dequant_chunk<Q>(pk[k], lo, hi, a);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                     rbase + static_cast<uint32_t>(c * 16)),
                                 "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w)
                                 : "memory");
                }
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (threadIdx.x == 0) {
            bulk_store(m.wq + row0 * m.cols, smem_addr(buf),
                       static_cast<uint32_t>(nrows * m.cols * 2));
            bulk_commit();
        }
    }
    if (threadIdx.x == 0) bulk_wait_all();
}

template <int Q, bool VEC, int CAP>
__global__ void __launch_bounds__(kThreads)
dequant_units_kernel(const __grid_constant__ MatBatch<CAP> p) {
    constexpr int B = Traits<Q>::bits;
    constexpr uint32_t mask = (1u << B) - 1u;
    int mi = 0;
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x) {
        mi = find_matrix(p, mi, u);
        const MatDesc& m = p.m[mi];
        const int tl = m.tpr_log2;
        const int tpr = 1 << tl;
        const int lane = threadIdx.x & (tpr - 1);
        const int rpb = kThreads >> tl;
        const int64_t row = (u - m.unit_begin) * rpb + (threadIdx.x >> tl);
        if (row >= m.rows) continue;
        const float a = __ldg(m.alpha + row);
        const uint8_t* src = m.packed + row * (m.cols * B / 8);
        uint16_t* dst = m.wq + row * m.cols;
        if constexpr (VEC) {
            // lane l decodes chunks l, l + tpr, ... of 8 codes: each warp
            // store writes 512 contiguous bytes
            uint32_t lo = 0, hi = 0;
            if constexpr (B == 2) dequant_table<Q>(a, lo, hi);  // the 4 outputs, byte-planar
            constexpr int U = 4;
            const int64_t nch = m.cols >> 3;
            for (int64_t ch = lane; ch < nch; ch += U * tpr) {
                uint32_t pk[U];
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int64_t c = ch + k * tpr;
                    if (c < nch) {
                        if constexpr (B == 2)
                            pk[k] = ld_stream(reinterpret_cast<const unsigned short*>(src + c * 2));
                        else
                            pk[k] = ld_stream(reinterpret_cast<const unsigned int*>(src + c * 4));
                    }
                }
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int64_t c = ch + k * tpr;
                    if (c < nch)
                        st_stream(reinterpret_cast<uint4*>(dst + c * 8),
                                  dequant_chunk<Q>(pk[k], lo, hi, a));
                }
            }
        } else {  // element path: groups of 8 codes
            const int64_t nch = (m.cols + 7) >> 3;
            for (int64_t ch = lane; ch < nch; ch += tpr) {
                const int n = tail_n(m.cols, ch);
                uint32_t pk = 0;
#pragma unroll
                for (int k = 0; k < B; ++k)  // B bytes hold 8 codes
                    if (k * (8 / B) < n) pk |= static_cast<uint32_t>(src[ch * B + k]) << (8 * k);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const uint32_t hw = pack_bf16x2(
                        __fmul_rn(level_of_field<Q>((pk >> (B * i)) & mask), a),
                        __fmul_rn(level_of_field<Q>((pk >> (B * (i + 1))) & mask), a));
                    if (i < n) dst[ch * 8 + i] = static_cast<uint16_t>(hw);
                    if (i + 1 < n) dst[ch * 8 + i + 1] = static_cast<uint16_t>(hw >> 16);
                }
            }
        }
    }
}

// ------------------------------------------------ backward fused with AdamW
// fp32 factors of one AdamW step, formed on the host in double from the
// hyperparameters and rounded once (see pq_adamw_t in pq.h).
struct AdamK {
    float decay, b1, c1, b2, c2, inv_sbc2, step, eps;
    int32_t has_decay;
    int32_t pad_;
};

// AdamW on one parameter: p*decay (if any), m = b1*m + c1*g,
// v = b2*v + c2*(g*g), p -= step * m / (sqrt(v)*inv_sbc2 + eps); every
// step rounds on its own (IEEE square root and division).
__device__ __forceinline__ float adamw_update(const AdamK& k, float p, float g, float& m,
                                              float& v) {
    if (k.has_decay) p = __fmul_rn(p, k.decay);
    m = __fadd_rn(__fmul_rn(k.b1, m), __fmul_rn(k.c1, g));
    v = __fadd_rn(__fmul_rn(k.b2, v), __fmul_rn(k.c2, __fmul_rn(g, g)));
    const float den = __fadd_rn(__fmul_rn(__fsqrt_rn(v), k.inv_sbc2), k.eps);
    return __fsub_rn(p, __fmul_rn(k.step, __fdiv_rn(m, den)));
}

struct AdamDesc {
    float* w;              // shadow weights, updated in place
    float* alpha;          // scales, updated in place
    const uint16_t* g;     // upstream gradient dWq (bf16)
    float* m_w;            // first moments of w
    float* v_w;            // second moments of w
    float* m_a;            // first moments of alpha
    float* v_a;            // second moments of alpha
    float* dalpha;         // d(alpha) out (nullable)
    int64_t rows;
    int64_t cols;
    int64_t unit_begin;
    float grad_scale;
    int32_t tpr_log2;
};

struct AdamBatch {
    BatchT<AdamDesc> b;
    AdamK kw;  // weights
    AdamK ka;  // scales
};

template <int Q, bool VEC>
__global__ void __launch_bounds__(kThreads, 3)
bwd_adamw_units_kernel(const __grid_constant__ AdamBatch P) {
    const BatchT<AdamDesc>& p = P.b;
    __shared__ double warp_sum[2][kThreads / 32];
    int mi = 0, prev_mi = 0, parity = 0;
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x, parity ^= 1) {
        mi = find_matrix(p, mi, u);
        if (mi != prev_mi) __syncthreads();
        prev_mi = mi;
        const AdamDesc& m = p.m[mi];
        const int tl = m.tpr_log2;
        const int tpr = 1 << tl;
        const int lane = threadIdx.x & (tpr - 1);
        const int rsub = threadIdx.x >> tl;
        const int64_t row = (u - m.unit_begin) * (kThreads >> tl) + rsub;
        const int64_t nch = (m.cols + 7) >> 3;
        double acc = 0.0;
        if (row < m.rows) {
            // plain load: alpha is written by this kernel (after every
            // thread of the row has read it)
            const RowScale a = row_scale(m.alpha[row]);
            float* wr = m.w + row * m.cols;
            const uint16_t* gr = m.g + row * m.cols;
            float* mr = m.m_w + row * m.cols;
            float* vr = m.v_w + row * m.cols;
            for (int64_t ch = lane; ch < nch; ch += tpr) {
                const int n = VEC ? 8 : tail_n(m.cols, ch);
                float wv[8], mv[8], vv[8], d[8];
                uint32_t gw[4];
                if constexpr (VEC) {
                    load8(wr + ch * 8, wv);
                    load_g8(gr + ch * 8, gw);
                    load8(mr + ch * 8, mv);
                    load8(vr + ch * 8, vv);
                } else {
                    load8_tail(wr + ch * 8, n, wv);
                    load_g8_tail(gr + ch * 8, n, gw);
                    load8_tail(mr + ch * 8, n, mv);
                    load8_tail(vr + ch * 8, n, vv);
                }
                acc = bwd_chunk<Q>(wv, gw, a, d, acc);
#pragma unroll
                for (int i = 0; i < 8; ++i) wv[i] = adamw_update(P.kw, wv[i], d[i], mv[i], vv[i]);
                if constexpr (VEC) {
                    store8(wr + ch * 8, wv);
                    store8(mr + ch * 8, mv);
                    store8(vr + ch * 8, vv);
                } else {
                    store8_tail(wr + ch * 8, n, wv);
                    store8_tail(mr + ch * 8, n, mv);
                    store8_tail(vr + ch * 8, n, vv);
                }
            }
        }
        const int seg = tpr < 32 ? tpr : 32;
        for (int off = seg >> 1; off > 0; off >>= 1)
            acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off, seg));
        if (tpr > 32) {
            if ((threadIdx.x & 31) == 0) warp_sum[parity][threadIdx.x >> 5] = acc;
            group_barrier(1 + rsub, tpr);
            if (lane == 0) {
                const int w0 = threadIdx.x >> 5;
                double t = warp_sum[parity][w0];
                for (int k = 1; k < (tpr >> 5); ++k) t = __dadd_rn(t, warp_sum[parity][w0 + k]);
                acc = t;
            }
        }
        if (lane == 0 && row < m.rows) {
            const float da = static_cast<float>(__dmul_rn(acc, static_cast<double>(m.grad_scale)));
            if (m.dalpha) m.dalpha[row] = da;
            float ma = m.m_a[row], va = m.v_a[row];
            m.alpha[row] = adamw_update(P.ka, m.alpha[row], da, ma, va);
            m.m_a[row] = ma;
            m.v_a[row] = va;
        }
    }
}

// ------------------------------- reduce-scatter fused with backward + AdamW
// One rank's row shards: the upstream gradient of each shard row is summed
// over the n_src replicas' bf16 gradients (buffers of identical layout,
// local or on peer GPUs), in source order in fp32, times grad_mult; then the
// backward and AdamW of bwd_adamw_units_kernel.
constexpr int kMaxSources = 16;

struct ShardDesc {
    float* w;
    float* alpha;
    float* m_w;
    float* v_w;
    float* m_a;
    float* v_a;
    float* dalpha;
    int64_t rows;
    int64_t cols;
    int64_t g_offset;      // element offset of row 0 in every source buffer
    int64_t unit_begin;
    float grad_scale;
    int32_t tpr_log2;
};

struct ReduceBatch {
    BatchT<ShardDesc> b;
    const uint16_t* src[kMaxSources];
    int32_t n_src;
    float grad_mult;
    AdamK kw;
    AdamK ka;
};

template <int Q, bool VEC>
__global__ void __launch_bounds__(kThreads, PQ_RED_MIN_CTAS)
reduce_bwd_adamw_units_kernel(const __grid_constant__ ReduceBatch P) {
    const BatchT<ShardDesc>& p = P.b;
    __shared__ double warp_sum[2][kThreads / 32];
    int mi = 0, prev_mi = 0, parity = 0;
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x, parity ^= 1) {
        mi = find_matrix(p, mi, u);
        if (mi != prev_mi) __syncthreads();
        prev_mi = mi;
        const ShardDesc& m = p.m[mi];
        const int tl = m.tpr_log2;
        const int tpr = 1 << tl;
        const int lane = threadIdx.x & (tpr - 1);
        const int rsub = threadIdx.x >> tl;
        const int64_t row = (u - m.unit_begin) * (kThreads >> tl) + rsub;
        const int64_t nch = (m.cols + 7) >> 3;
        double acc = 0.0;
        if (row < m.rows) {
            const RowScale a = row_scale(m.alpha[row]);  // plain load: written below
            float* wr = m.w + row * m.cols;
            float* mr = m.m_w + row * m.cols;
            float* vr = m.v_w + row * m.cols;
            const int64_t goff = m.g_offset + row * m.cols;
            for (int64_t ch = lane; ch < nch; ch += tpr) {
                const int n = VEC ? 8 : tail_n(m.cols, ch);
                float wv[8], mv[8], vv[8], gs[8], d[8];
                if constexpr (VEC) {
                    load8(wr + ch * 8, wv);
                    load8(mr + ch * 8, mv);
                    load8(vr + ch * 8, vv);
                } else {
                    load8_tail(wr + ch * 8, n, wv);
                    load8_tail(mr + ch * 8, n, mv);
                    load8_tail(vr + ch * 8, n, vv);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) gs[i] = 0.0f;
#pragma unroll 4
                for (int k = 0; k < P.n_src; ++k) {
                    uint32_t gw[4];
                    if constexpr (VEC) load_g8(P.src[k] + goff + ch * 8, gw);
                    else load_g8_tail(P.src[k] + goff + ch * 8, n, gw);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        gs[i] = __fadd_rn(gs[i], (i & 1) ? __uint_as_float(gw[i / 2] & 0xFFFF0000u)
                                                         : __uint_as_float(gw[i / 2] << 16));
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) gs[i] = __fmul_rn(gs[i], P.grad_mult);
                acc = bwd_chunk_f32<Q>(wv, gs, a, d, acc);
#pragma unroll
                for (int i = 0; i < 8; ++i) wv[i] = adamw_update(P.kw, wv[i], d[i], mv[i], vv[i]);
                if constexpr (VEC) {
                    store8(wr + ch * 8, wv);
                    store8(mr + ch * 8, mv);
                    store8(vr + ch * 8, vv);
                } else {
                    store8_tail(wr + ch * 8, n, wv);
                    store8_tail(mr + ch * 8, n, mv);
                    store8_tail(vr + ch * 8, n, vv);
                }
            }
        }
        const int seg = tpr < 32 ? tpr : 32;
        for (int off = seg >> 1; off > 0; off >>= 1)
            acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off, seg));
        if (tpr > 32) {
            if ((threadIdx.x & 31) == 0) warp_sum[parity][threadIdx.x >> 5] = acc;
            group_barrier(1 + rsub, tpr);
            if (lane == 0) {
                const int w0 = threadIdx.x >> 5;
                double t = warp_sum[parity][w0];
                for (int k = 1; k < (tpr >> 5); ++k) t = __dadd_rn(t, warp_sum[parity][w0 + k]);
                acc = t;
            }
        }
        if (lane == 0 && row < m.rows) {
            const float da = static_cast<float>(__dmul_rn(acc, static_cast<double>(m.grad_scale)));
            if (m.dalpha) m.dalpha[row] = da;
            float ma = m.m_a[row], va = m.v_a[row];
            m.alpha[row] = adamw_update(P.ka, m.alpha[row], da, ma, va);
            m.m_a[row] = ma;
            m.v_a[row] = va;
        }
    }
}

// --------------------------------------------------------------- host side
static thread_local int g_last_cuda_error = 0;

static int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    return dev;
}

static int sm_count() {
    static int cached[64] = {0};
    const int dev = current_device();
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

// Threads per row: a power of two, 1..256, giving each thread about
// PQ_CHUNKS_PER_THREAD chunks of 8 weights of its row.
static inline int choose_tpr_log2_for(int64_t nch, int chunks_per_thread) {
    const int l = ilog2_ceil((nch + chunks_per_thread - 1) / chunks_per_thread);
    return l > 8 ? 8 : l;
}

static inline int choose_tpr_log2(int64_t cols) {
    return choose_tpr_log2_for((cols + 7) / 8, PQ_CHUNKS_PER_THREAD);
}

// Row groups of the backward kernels (one row per group: a row's d(alpha)
// is reduced inside its CTA). A matrix with too few rows to give every SM
// a unit takes wider groups (up to one thread per chunk of a row), so its
// chunks spread over more CTAs instead of queueing on a few threads.
static inline int bwd_tpr_log2(int64_t rows, int64_t cols) {
    const int64_t nch = (cols + 7) / 8;
    int l = choose_tpr_log2(cols);
    const int lmax = choose_tpr_log2_for(nch, 1);
    while (l < lmax && (rows + (kThreads >> l) - 1) / (kThreads >> l) < sm_count()) ++l;
    return l;
}

static pq_status_t cuda_status(cudaError_t e) {
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

// Calls f.template operator()<Q>() for the runtime quantizer q.
template <typename F>
static bool dispatch_q(int q, F&& f) {
    switch (q) {
        case PQ_BINARY: f.template operator()<PQ_BINARY>(); return true;
        case PQ_TERNARY: f.template operator()<PQ_TERNARY>(); return true;
        case PQ_SEQ2: f.template operator()<PQ_SEQ2>(); return true;
        case PQ_SEQ2_B: f.template operator()<PQ_SEQ2_B>(); return true;
        case PQ_LSQ2: f.template operator()<PQ_LSQ2>(); return true;
        case PQ_LSQ3: f.template operator()<PQ_LSQ3>(); return true;
        case PQ_LSQ4: f.template operator()<PQ_LSQ4>(); return true;
        default: return false;
    }
}

// Persistent grid size of one kernel, from its occupancy (once per device).
template <typename K>
static int64_t persistent_ctas(K kernel, int* cache) {
    const int dev = current_device();
    if (cache[dev] == 0) {
        int per_sm = PQ_CTAS_PER_SM;
        if (per_sm <= 0 &&
            (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) !=
                 cudaSuccess || per_sm <= 0))
            per_sm = 4;
        cache[dev] = per_sm * sm_count();
    }
    return cache[dev];
}

// The descriptors of a batch that fits the small parameter block, copied
// into it (host side, per thread).
static const MatBatch<kSmallBatch>& small_batch(const Batch& b) {
    static thread_local MatBatch<kSmallBatch> sb;
    sb.n = b.n;
    sb.pad_ = 0;
    sb.total_units = b.total_units;
    for (int i = 0; i < b.n; ++i) sb.m[i] = b.m[i];
    return sb;
}

template <int Q, bool VEC, bool WQ, bool PACK, int CAP>
static void launch_fwd_cap(const MatBatch<CAP>& b, cudaStream_t s) {
    static int cache[64] = {0};
    auto k = fwd_units_kernel<Q, VEC, WQ, PACK, CAP>;
    const int64_t ctas = persistent_ctas(k, cache);
    const unsigned grid = static_cast<unsigned>(b.total_units < ctas ? b.total_units : ctas);
    k<<<grid, kThreads, 0, s>>>(b);
    pqc::count_launch();
}

template <int Q, bool VEC, bool WQ, bool PACK>
static void launch_fwd(const Batch& b, cudaStream_t s) {
    if (b.n <= kSmallBatch) launch_fwd_cap<Q, VEC, WQ, PACK, kSmallBatch>(small_batch(b), s);
    else launch_fwd_cap<Q, VEC, WQ, PACK, kMaxBatch>(b, s);
}

template <int Q, bool VEC, int CAP>
static void launch_bwd_cap(const MatBatch<CAP>& b, cudaStream_t s) {
    static int cache[64] = {0};
    auto k = bwd_units_kernel<Q, VEC, CAP>;
    const int64_t ctas = persistent_ctas(k, cache);
    const unsigned grid = static_cast<unsigned>(b.total_units < ctas ? b.total_units : ctas);
    k<<<grid, kThreads, 0, s>>>(b);
    pqc::count_launch();
}

template <int Q, bool VEC>
static void launch_bwd(const Batch& b, cudaStream_t s) {
    if (b.n <= kSmallBatch) launch_bwd_cap<Q, VEC, kSmallBatch>(small_batch(b), s);
    else launch_bwd_cap<Q, VEC, kMaxBatch>(b, s);
}

template <int Q, bool VEC, int CAP>
static void launch_dequant_cap(const MatBatch<CAP>& b, cudaStream_t s) {
    static int cache[64] = {0};
    auto k = dequant_units_kernel<Q, VEC, CAP>;
    const int64_t ctas = persistent_ctas(k, cache);
    const unsigned grid = static_cast<unsigned>(b.total_units < ctas ? b.total_units : ctas);
    k<<<grid, kThreads, 0, s>>>(b);
    pqc::count_launch();
}

template <int Q, bool VEC>
static void launch_dequant(const Batch& b, cudaStream_t s) {
    if (b.n <= kSmallBatch) launch_dequant_cap<Q, VEC, kSmallBatch>(small_batch(b), s);
    else launch_dequant_cap<Q, VEC, kMaxBatch>(b, s);
}

template <int Q, int CAP>
static cudaError_t launch_dequant_bulk_cap(const MatBatch<CAP>& b, cudaStream_t s) {
    static int cache[64] = {0};
    static bool attr_set[64] = {false};
    auto k = dequant_bulk_kernel<Q, CAP>;
    constexpr int smem = 2 * kDeqBuf;
    const int dev = current_device();
    if (!attr_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    if (cache[dev] == 0) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, smem) !=
                cudaSuccess || per_sm <= 0)
            per_sm = 1;
        cache[dev] = per_sm * sm_count();
    }
    const int64_t ctas = cache[dev];
    const unsigned grid = static_cast<unsigned>(b.total_units < ctas ? b.total_units : ctas);
    k<<<grid, kThreads, smem, s>>>(b);
    pqc::count_launch();
    return cudaSuccess;
}

template <int Q>
static cudaError_t launch_dequant_bulk(const Batch& b, cudaStream_t s) {
    if (b.n <= kSmallBatch) return launch_dequant_bulk_cap<Q, kSmallBatch>(small_batch(b), s);
    return launch_dequant_bulk_cap<Q, kMaxBatch>(b, s);
}

// ------------------------------------------------------- validation
static bool fwd_vec_ok(const pq_matrix_t& m, int bits) {
    return m.cols % 8 == 0 && aligned(m.w, 32) &&
           (!m.wq_bf16_out || aligned(m.wq_bf16_out, 16)) &&
           (!m.packed_out || aligned(m.packed_out, bits == 2 ? 2 : 4));
}

static bool bwd_vec_ok(const pq_matrix_t& m) {
    return m.cols % 8 == 0 && aligned(m.w, 32) && aligned(m.g_bf16, 16) && aligned(m.dw_out, 32);
}

static pq_status_t check_fwd(int bits, const pq_matrix_t& m) {
    if (m.rows < 0 || m.cols < 0) return PQ_ERR_INVALID_ARG;
    if (m.packed_out && (m.cols % (8 / bits)) != 0) return PQ_ERR_INVALID_ARG;
    if (m.rows == 0 || m.cols == 0) return PQ_OK;
    if (!m.wq_bf16_out && !m.packed_out) return PQ_ERR_INVALID_ARG;
    if (!m.w || !m.alpha) return PQ_ERR_INVALID_ARG;
    return PQ_OK;
}

static pq_status_t check_bwd(const pq_matrix_t& m) {
    if (m.rows < 0 || m.cols < 0) return PQ_ERR_INVALID_ARG;
    if (m.rows == 0) return PQ_OK;
    if (!m.dalpha_out) return PQ_ERR_INVALID_ARG;
    if (m.cols == 0) return PQ_OK;
    if (!m.w || !m.alpha || !m.g_bf16 || !m.dw_out) return PQ_ERR_INVALID_ARG;
    return PQ_OK;
}

static void batch_reset(Batch& b) {
    b.n = 0;
    b.pad_ = 0;
    b.total_units = 0;
}

// Appends one matrix; col_splits > 1 splits each row block's columns into
// that many units (forward only).
static void batch_add(Batch& b, const pq_matrix_t& m, int tl, int col_splits) {
    MatDesc& d = b.m[b.n++];
    d.w = m.w;
    d.alpha = m.alpha;
    d.wq = m.wq_bf16_out;
    d.packed = m.packed_out;
    d.g = m.g_bf16;
    d.dw = m.dw_out;
    d.dalpha = m.dalpha_out;
    d.rows = m.rows;
    d.cols = m.cols;
    d.unit_begin = b.total_units;
    d.grad_scale = m.grad_scale;
    d.tpr_log2 = tl;
    d.col_splits = col_splits;
    d.pad_ = 0;
    const int64_t rpb = kThreads >> tl;
    b.total_units += (m.rows + rpb - 1) / rpb * col_splits;
}

// Forward over n matrices. Matrices are grouped by output kind (bf16 and
// packed, bf16 only, packed only) and by layout (vector or element path);
// each group goes out in launches of up to kMaxBatch descriptors.
static pq_status_t fwd_batch_impl(int q, int32_t n, const pq_matrix_t* mats, cudaStream_t s) {
    const int bits = code_bits_of(q);
    if (bits == 0 || n < 0 || (n > 0 && !mats)) return PQ_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        const pq_status_t st = check_fwd(bits, mats[i]);
        if (st != PQ_OK) return st;
    }
    static thread_local Batch b;
    bool launched = false;
    const int64_t fill = 2 * static_cast<int64_t>(sm_count());
    for (int cls = 0; cls < 6; ++cls) {
        const int kind = cls >> 1;   // 0: wq+packed, 1: wq only, 2: packed only
        const bool vec = (cls & 1) == 0;
        batch_reset(b);
        auto flush = [&]() {
            if (b.n == 0) return;
            launched = true;
            dispatch_q(q, [&]<int Q>() {
                if (vec) {
                    if (kind == 0) launch_fwd<Q, true, true, true>(b, s);
                    else if (kind == 1) launch_fwd<Q, true, true, false>(b, s);
                    else launch_fwd<Q, true, false, true>(b, s);
                } else {
                    if (kind == 0) launch_fwd<Q, false, true, true>(b, s);
                    else if (kind == 1) launch_fwd<Q, false, true, false>(b, s);
                    else launch_fwd<Q, false, false, true>(b, s);
                }
            });
            batch_reset(b);
        };
        for (int32_t i = 0; i < n; ++i) {
            const pq_matrix_t& m = mats[i];
            if (m.rows == 0 || m.cols == 0) continue;
            const int k = (m.wq_bf16_out && m.packed_out) ? 0 : (m.wq_bf16_out ? 1 : 2);
            if (k != kind || fwd_vec_ok(m, bits) != vec) continue;
            const int tl = choose_tpr_log2_for((m.cols + 7) / 8, PQ_FWD_CHUNKS_PER_THREAD);
            const int64_t tpr = int64_t{1} << tl;
            const int64_t rpb = kThreads >> tl;
            const int64_t row_blocks = (m.rows + rpb - 1) / rpb;
            int64_t splits = 1;
            if (row_blocks < fill) {  // few rows: split the columns too
                const int64_t nch = (m.cols + 7) / 8;
                const int64_t max_splits = (nch + 2 * tpr - 1) / (2 * tpr);
                splits = (fill + row_blocks - 1) / row_blocks;
                if (splits > max_splits) splits = max_splits;
                if (splits < 1) splits = 1;
            }
            if (b.n == kMaxBatch) flush();
            batch_add(b, m, tl, static_cast<int>(splits));
        }
        flush();
    }
    return launched ? cuda_status(cudaGetLastError()) : PQ_OK;
}

static pq_status_t bwd_batch_impl(int q, int32_t n, const pq_matrix_t* mats, cudaStream_t s) {
    if (code_bits_of(q) == 0 || n < 0 || (n > 0 && !mats)) return PQ_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        const pq_status_t st = check_bwd(mats[i]);
        if (st != PQ_OK) return st;
    }
    static thread_local Batch b;
    bool launched = false;
    for (int32_t i = 0; i < n; ++i) {  // rows without columns: d(alpha) = 0
        const pq_matrix_t& m = mats[i];
        if (m.rows > 0 && m.cols == 0) {
            launched = true;
            const pq_status_t st = cuda_status(cudaMemsetAsync(
                m.dalpha_out, 0, static_cast<size_t>(m.rows) * sizeof(float), s));
            if (st != PQ_OK) return st;
        }
    }
    for (int cls = 0; cls < 2; ++cls) {
        const bool vec = cls == 0;
        batch_reset(b);
        auto flush = [&]() {
            if (b.n == 0) return;
            launched = true;
            dispatch_q(q, [&]<int Q>() {
                if (vec) launch_bwd<Q, true>(b, s);
                else launch_bwd<Q, false>(b, s);
            });
            batch_reset(b);
        };
        for (int32_t i = 0; i < n; ++i) {
            const pq_matrix_t& m = mats[i];
            if (m.rows == 0 || m.cols == 0 || bwd_vec_ok(m) != vec) continue;
            if (b.n == kMaxBatch) flush();
            batch_add(b, m, bwd_tpr_log2(m.rows, m.cols), 1);
        }
        flush();
    }
    return launched ? cuda_status(cudaGetLastError()) : PQ_OK;
}

// Dequantization over n matrices (packed_out is read, wq_bf16_out written).
static pq_status_t dequant_batch_impl(int q, int32_t n, const pq_matrix_t* mats, cudaStream_t s) {
    const int bits = code_bits_of(q);
    if (bits == 0 || n < 0 || (n > 0 && !mats)) return PQ_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        const pq_matrix_t& m = mats[i];
        if (m.rows < 0 || m.cols < 0 || m.cols % (8 / bits) != 0) return PQ_ERR_INVALID_ARG;
        if (m.rows > 0 && m.cols > 0 && (!m.packed_out || !m.alpha || !m.wq_bf16_out))
            return PQ_ERR_INVALID_ARG;
    }
    static thread_local Batch b;
    bool launched = false;
    cudaError_t err = cudaSuccess;
    // classes: 0 staged bulk stores (vector layout, a row block's output fits
    // one staging buffer), 1 vector layout, 2 element path
    for (int cls = 0; cls < 3; ++cls) {
        if (cls == 0 && !PQ_DEQ_BULK) continue;
        batch_reset(b);
        auto flush = [&]() {
            if (b.n == 0) return;
            launched = true;
            dispatch_q(q, [&]<int Q>() {
                if (cls == 0) {
                    const cudaError_t e = launch_dequant_bulk<Q>(b, s);
                    if (e != cudaSuccess) err = e;
                } else if (cls == 1) {
                    launch_dequant<Q, true>(b, s);
                } else {
                    launch_dequant<Q, false>(b, s);
                }
            });
            batch_reset(b);
        };
        for (int32_t i = 0; i < n; ++i) {
            const pq_matrix_t& m = mats[i];
            if (m.rows == 0 || m.cols == 0) continue;
            const bool v = m.cols % 8 == 0 && aligned(m.packed_out, bits == 2 ? 2 : 4) &&
                           aligned(m.wq_bf16_out, 16);
            const int bulk_tl = choose_tpr_log2_for((m.cols + 7) / 8, kDeqChunks);
            const bool bulk = PQ_DEQ_BULK && v && (int64_t{kDeqChunks} << bulk_tl) * 8 >= m.cols;
            const int c = bulk ? 0 : (v ? 1 : 2);
            if (c != cls) continue;
            if (b.n == kMaxBatch) flush();
            batch_add(b, m, cls == 0 ? bulk_tl : choose_tpr_log2(m.cols), 1);
        }
        flush();
    }
    if (err != cudaSuccess) return cuda_status(err);
    return launched ? cuda_status(cudaGetLastError()) : PQ_OK;
}

static AdamK adamw_consts(const pq_adamw_t& h) {
    AdamK k;
    const double t = static_cast<double>(h.step);
    k.decay = static_cast<float>(1.0 - h.lr * h.weight_decay);
    k.has_decay = h.weight_decay != 0.0;
    k.b1 = static_cast<float>(h.beta1);
    k.c1 = static_cast<float>(1.0 - h.beta1);
    k.b2 = static_cast<float>(h.beta2);
    k.c2 = static_cast<float>(1.0 - h.beta2);
    k.inv_sbc2 = static_cast<float>(1.0 / sqrt(1.0 - pow(h.beta2, t)));
    k.step = static_cast<float>(h.lr / (1.0 - pow(h.beta1, t)));
    k.eps = static_cast<float>(h.eps);
    k.pad_ = 0;
    return k;
}

static bool adamw_ok(const pq_adamw_t* h) {
    return h && h->step >= 1 && h->beta1 >= 0.0 && h->beta1 < 1.0 && h->beta2 >= 0.0 &&
           h->beta2 < 1.0 && h->eps > 0.0 && h->lr >= 0.0;
}

template <int Q, bool VEC>
static void launch_bwd_adamw(const AdamBatch& b, cudaStream_t s) {
    static int cache[64] = {0};
    auto k = bwd_adamw_units_kernel<Q, VEC>;
    const int64_t ctas = persistent_ctas(k, cache);
    const unsigned grid = static_cast<unsigned>(b.b.total_units < ctas ? b.b.total_units : ctas);
    k<<<grid, kThreads, 0, s>>>(b);
    pqc::count_launch();
}

static pq_status_t bwd_adamw_impl(int q, int32_t n, const pq_adamw_matrix_t* mats,
                                  const pq_adamw_t* hw, const pq_adamw_t* ha, cudaStream_t s) {
    if (code_bits_of(q) == 0 || n < 0 || (n > 0 && !mats)) return PQ_ERR_INVALID_ARG;
    if (!adamw_ok(hw) || !adamw_ok(ha)) return PQ_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        const pq_adamw_matrix_t& m = mats[i];
        if (m.rows < 0 || m.cols < 0) return PQ_ERR_INVALID_ARG;
        if (m.rows == 0) continue;
        if (!m.alpha || !m.m_alpha || !m.v_alpha) return PQ_ERR_INVALID_ARG;
        if (m.cols > 0 && (!m.w || !m.g_bf16 || !m.m_w || !m.v_w)) return PQ_ERR_INVALID_ARG;
    }
    static thread_local AdamBatch b;
    b.kw = adamw_consts(*hw);
    b.ka = adamw_consts(*ha);
    bool launched = false;
    for (int cls = 0; cls < 2; ++cls) {
        const bool vec = cls == 0;
        b.b.n = 0;
        b.b.pad_ = 0;
        b.b.total_units = 0;
        auto flush = [&]() {
            if (b.b.n == 0) return;
            launched = true;
            dispatch_q(q, [&]<int Q>() {
                if (vec) launch_bwd_adamw<Q, true>(b, s);
                else launch_bwd_adamw<Q, false>(b, s);
            });
            b.b.n = 0;
            b.b.total_units = 0;
        };
        for (int32_t i = 0; i < n; ++i) {
            const pq_adamw_matrix_t& m = mats[i];
            if (m.rows == 0) continue;
            // rows without columns still take an AdamW step on alpha with
            // d(alpha) = 0: they go through the element path
            const bool v = m.cols > 0 && m.cols % 8 == 0 && aligned(m.w, 32) &&
                           aligned(m.g_bf16, 16) && aligned(m.m_w, 32) && aligned(m.v_w, 32);
            if (v != vec) continue;
            if (b.b.n == kMaxBatch) flush();
            AdamDesc& d = b.b.m[b.b.n++];
            d.w = m.w;
            d.alpha = m.alpha;
            d.g = m.g_bf16;
            d.m_w = m.m_w;
            d.v_w = m.v_w;
            d.m_a = m.m_alpha;
            d.v_a = m.v_alpha;
            d.dalpha = m.dalpha_out;
            d.rows = m.rows;
            d.cols = m.cols;
            d.unit_begin = b.b.total_units;
            d.grad_scale = m.grad_scale;
            d.tpr_log2 = bwd_tpr_log2(m.rows, m.cols);
            b.b.total_units += (m.rows + (kThreads >> d.tpr_log2) - 1) / (kThreads >> d.tpr_log2);
        }
        flush();
    }
    return launched ? cuda_status(cudaGetLastError()) : PQ_OK;
}

template <int Q, bool VEC>
static void launch_reduce_bwd_adamw(const ReduceBatch& b, cudaStream_t s) {
    static int cache[64] = {0};
    auto k = reduce_bwd_adamw_units_kernel<Q, VEC>;
    const int64_t ctas = persistent_ctas(k, cache);
    const unsigned grid = static_cast<unsigned>(b.b.total_units < ctas ? b.b.total_units : ctas);
    k<<<grid, kThreads, 0, s>>>(b);
    pqc::count_launch();
}

static pq_status_t reduce_bwd_adamw_impl(int q, int32_t n_src, const uint16_t* const* srcs,
                                         float grad_mult, int32_t n, const pq_shard_t* sh,
                                         const pq_adamw_t* hw, const pq_adamw_t* ha,
                                         cudaStream_t s) {
    if (code_bits_of(q) == 0 || n < 0 || (n > 0 && !sh)) return PQ_ERR_INVALID_ARG;
    if (n_src < 1 || n_src > kMaxSources || !srcs) return PQ_ERR_INVALID_ARG;
    if (!adamw_ok(hw) || !adamw_ok(ha)) return PQ_ERR_INVALID_ARG;
    bool src_aligned = true;
    for (int k = 0; k < n_src; ++k) {
        if (!srcs[k]) return PQ_ERR_INVALID_ARG;
        src_aligned = src_aligned && aligned(srcs[k], 16);
    }
    for (int32_t i = 0; i < n; ++i) {
        const pq_shard_t& m = sh[i];
        if (m.rows < 0 || m.cols < 0 || m.g_offset < 0) return PQ_ERR_INVALID_ARG;
        if (m.rows == 0) continue;
        if (!m.alpha || !m.m_alpha || !m.v_alpha) return PQ_ERR_INVALID_ARG;
        if (m.cols > 0 && (!m.w || !m.m_w || !m.v_w)) return PQ_ERR_INVALID_ARG;
    }
    static thread_local ReduceBatch b;
    for (int k = 0; k < kMaxSources; ++k) b.src[k] = k < n_src ? srcs[k] : nullptr;
    b.n_src = n_src;
    b.grad_mult = grad_mult;
    b.kw = adamw_consts(*hw);
    b.ka = adamw_consts(*ha);
    bool launched = false;
    for (int cls = 0; cls < 2; ++cls) {
        const bool vec = cls == 0;
        b.b.n = 0;
        b.b.pad_ = 0;
        b.b.total_units = 0;
        auto flush = [&]() {
            if (b.b.n == 0) return;
            launched = true;
            dispatch_q(q, [&]<int Q>() {
                if (vec) launch_reduce_bwd_adamw<Q, true>(b, s);
                else launch_reduce_bwd_adamw<Q, false>(b, s);
            });
            b.b.n = 0;
            b.b.total_units = 0;
        };
        for (int32_t i = 0; i < n; ++i) {
            const pq_shard_t& m = sh[i];
            if (m.rows == 0) continue;
            const bool v = src_aligned && m.cols > 0 && m.cols % 8 == 0 && m.g_offset % 8 == 0 &&
                           aligned(m.w, 32) && aligned(m.m_w, 32) && aligned(m.v_w, 32);
            if (v != vec) continue;
            if (b.b.n == kMaxBatch) flush();
            ShardDesc& d = b.b.m[b.b.n++];
            d.w = m.w;
            d.alpha = m.alpha;
            d.m_w = m.m_w;
            d.v_w = m.v_w;
            d.m_a = m.m_alpha;
            d.v_a = m.v_alpha;
            d.dalpha = m.dalpha_out;
            d.rows = m.rows;
            d.cols = m.cols;
            d.g_offset = m.g_offset;
            d.unit_begin = b.b.total_units;
            d.grad_scale = m.grad_scale;
            d.tpr_log2 = bwd_tpr_log2(m.rows, m.cols);
            b.b.total_units += (m.rows + (kThreads >> d.tpr_log2) - 1) / (kThreads >> d.tpr_log2);
        }
        flush();
    }
    return launched ? cuda_status(cudaGetLastError()) : PQ_OK;
}

}  // namespace pq

using namespace pq;

extern "C" {

pq_status_t pq_fakequant_fwd(pq_quant_t q, int64_t rows, int64_t cols, const float* w,
                             const float* alpha, uint16_t* wq_bf16_out, uint8_t* packed_out,
                             void* stream) {
    if (!wq_bf16_out && rows > 0 && cols > 0) return PQ_ERR_INVALID_ARG;
    pq_matrix_t m = {};
    m.rows = rows;
    m.cols = cols;
    m.w = w;
    m.alpha = alpha;
    m.wq_bf16_out = wq_bf16_out;
    m.packed_out = packed_out;
    return fwd_batch_impl(q, 1, &m, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_pack_codes(pq_quant_t q, int64_t rows, int64_t cols, const float* w,
                          const float* alpha, uint8_t* packed_out, void* stream) {
    if (!packed_out && rows > 0 && cols > 0) return PQ_ERR_INVALID_ARG;
    pq_matrix_t m = {};
    m.rows = rows;
    m.cols = cols;
    m.w = w;
    m.alpha = alpha;
    m.packed_out = packed_out;
    return fwd_batch_impl(q, 1, &m, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_fakequant_bwd(pq_quant_t q, int64_t rows, int64_t cols, const float* w,
                             const float* alpha, const uint16_t* g_bf16, float* dw_out,
                             float* dalpha_out, float grad_scale, void* stream) {
    pq_matrix_t m = {};
    m.rows = rows;
    m.cols = cols;
    m.w = w;
    m.alpha = alpha;
    m.g_bf16 = g_bf16;
    m.dw_out = dw_out;
    m.dalpha_out = dalpha_out;
    m.grad_scale = grad_scale;
    return bwd_batch_impl(q, 1, &m, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_scaled_weights(int64_t rows, int64_t cols, const float* w, const float* alpha,
                              float* x_out, void* stream) {
    if (rows < 0 || cols < 0) return PQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return PQ_OK;
    if (!w || !alpha || !x_out) return PQ_ERR_INVALID_ARG;
    const int64_t nch = (cols + 7) / 8;
    int64_t gx = (nch + kThreads - 1) / kThreads;
    if (gx > 1024) gx = 1024;
    const int64_t gy = rows < 65535 ? rows : 65535;
    scaled_weights_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kThreads,
                            0, static_cast<cudaStream_t>(stream)>>>(w, alpha, x_out, rows, cols);
    pqc::count_launch();
    return cuda_status(cudaGetLastError());
}

pq_status_t pq_dequant_codes(pq_quant_t q, int64_t rows, int64_t cols, const uint8_t* packed,
                             const float* alpha, uint16_t* wq_bf16_out, void* stream) {
    pq_matrix_t m = {};
    m.rows = rows;
    m.cols = cols;
    m.alpha = alpha;
    m.packed_out = const_cast<uint8_t*>(packed);
    m.wq_bf16_out = wq_bf16_out;
    return dequant_batch_impl(q, 1, &m, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_dequant_codes_batch(pq_quant_t q, int32_t n, const pq_matrix_t* mats,
                                   void* stream) {
    return dequant_batch_impl(q, n, mats, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_fakequant_bwd_adamw(pq_quant_t q, int32_t n, const pq_adamw_matrix_t* mats,
                                   const pq_adamw_t* hp_w, const pq_adamw_t* hp_alpha,
                                   void* stream) {
    return bwd_adamw_impl(q, n, mats, hp_w, hp_alpha, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_reduce_bwd_adamw(pq_quant_t q, int32_t n_src, const uint16_t* const* g_sources,
                                float grad_mult, int32_t n, const pq_shard_t* shards,
                                const pq_adamw_t* hp_w, const pq_adamw_t* hp_alpha, void* stream) {
    return reduce_bwd_adamw_impl(q, n_src, g_sources, grad_mult, n, shards, hp_w, hp_alpha,
                                 static_cast<cudaStream_t>(stream));
}

pq_status_t pq_fakequant_fwd_batch(pq_quant_t q, int32_t n, const pq_matrix_t* mats,
                                   void* stream) {
    return fwd_batch_impl(q, n, mats, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_fakequant_bwd_batch(pq_quant_t q, int32_t n, const pq_matrix_t* mats,
                                   void* stream) {
    return bwd_batch_impl(q, n, mats, static_cast<cudaStream_t>(stream));
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

int64_t pq_launch_count(void) { return pqc::launches.load(std::memory_order_relaxed); }

}  // extern "C"
