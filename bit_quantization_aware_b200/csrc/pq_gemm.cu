// Weight-only low-bit matmul on sm_100a tensor cores (tcgen05 + TMEM).
//
//   Y[m][n] = sum_k X[m][k] * level(code[n][k]) * alpha[n]
//
// X: bf16 [M, K] activations (M <= 128, a decode-sized batch); codes: the
// forward's packed 2-bit codes [N, K/4]; alpha: fp32 [N]; Y: bf16 [M, N].
// Every 2-bit level is a small integer numerator times a per-quantizer
// factor (SEQ2 (2c+1)/4, SEQ2_B (2c+1)/3, ternary 2c/3, LSQ2 and binary c),
// so the weight tile is decoded to exact bf16 numerators and the factor
// times alpha scales the fp32 accumulator in the epilogue.
//
// The weights are the wide operand: each CTA tile is 128 output features
// (the MMA's M) by NT batch columns (the MMA's N, NT >= M), accumulated in
// TMEM over K. A persistent CTA of 4 warps walks (feature block, K segment)
// units; per pipeline stage of 128 K, every thread decodes its feature row's
// 128 codes (32 bytes) into the 128B-swizzled K-major shared-memory layout
// through a byte-permute table, the activations arrive by cp.async, and
// thread 0 issues 8 tcgen05.mma (K = 16 each) and commits them to the
// stage's mbarrier. Split-K partial sums go to a caller workspace; the last
// CTA of a feature block adds them in segment order (deterministic).
//
// Every mbarrier wait is bounded: on giving up, the kernel records a device
// status, waits (bounded) for its own MMAs, frees its TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <stdint.h>

#include <atomic>

#include "pq.h"

namespace pqg {

constexpr int kThreads = 128;         // 4 warps = the 128 TMEM lanes
constexpr int kBlockN = 128;          // features per tile (MMA M)
constexpr int kStageK = 128;          // K per stage (two 64-wide swizzle atoms)
constexpr int kStages = 3;
constexpr uint32_t kMaxSpins = 1u << 22;

// nonzero after a bounded wait gave up (read by pq_device_status)
__device__ int g_status = 0;

struct GemmParams {
    const uint16_t* x;      // [M, K] bf16
    const uint8_t* codes;   // [N, K/4]
    const float* alpha;     // [N]
    uint16_t* y;            // [M, N] bf16
    float* partial;         // [S, M, N] fp32 (S > 1)
    int* counters;          // [ceil(N/128)] (S > 1), zero on entry
    int64_t m, n, k;
    int64_t kseg;           // K per segment (multiple of kStageK)
    int32_t splits;         // S
    int32_t nblocks;
    uint32_t table_lo;      // bf16 numerators of fields 0..3, low bytes
    uint32_t table_hi;      // ... high bytes
    float factor;           // level = numerator * factor
};

// ----------------------------------------------------------- primitives
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major, 128-byte swizzle shared-memory matrix descriptor: start >> 4,
// leading offset 16 B (unused for this layout), stride between 8-row
// groups 1024 B, descriptor version 1, layout type 2 (128B swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (uint64_t{1} << 16) |
           (uint64_t{1024 >> 4} << 32) | (uint64_t{1} << 46) | (uint64_t{2} << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, M = 128, N = nt.
__host__ __device__ constexpr uint32_t idesc_bf16(int nt) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nt >> 3) << 17) |
           (static_cast<uint32_t>(kBlockN >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     mbar)
                 : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

// Bounded wait for the given phase parity; false when it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    for (uint32_t i = 0; i < kMaxSpins; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    atomicExch(&g_status, 1);
    return false;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}

// 16 fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Fields of byte b (4 codes of 2 bits) moved to bits 0, 8, 16, 24.
__device__ __forceinline__ uint32_t spread2(uint32_t b) {
    return ((b & 0x33u) * 0x1001u | (b & 0xCCu) * 0x40040u) & 0x03030303u;
}

// 8 codes (16 bits) -> 8 bf16 numerators (4 words) via the byte-planar table.
__device__ __forceinline__ uint4 decode8(uint32_t h16, uint32_t lo, uint32_t hi) {
    const uint32_t t0 = spread2(h16 & 0xFFu);
    const uint32_t t1 = spread2(h16 >> 8);
    uint4 o;
    o.x = __byte_perm(lo, hi, t0 * 0x11u + 0x4040u);
    o.y = __byte_perm(lo, hi, (t0 >> 16) * 0x11u + 0x4040u);
    o.z = __byte_perm(lo, hi, t1 * 0x11u + 0x4040u);
    o.w = __byte_perm(lo, hi, (t1 >> 16) * 0x11u + 0x4040u);
    return o;
}

template <int NT>
struct Layout {
    static constexpr int kAtomA = kBlockN * 128;        // 128 rows x 128 B
    static constexpr int kAtomB = NT * 128;             // NT rows x 128 B
    static constexpr int kStage = 2 * kAtomA + 2 * kAtomB;
    static constexpr int kBarriers = kStages * kStage;  // offset of the barriers
    static constexpr int kBytes = kBarriers + 256 + 1024;  // + barriers, slack for alignment
    static constexpr uint32_t kCols = NT < 32 ? 32 : NT;   // TMEM columns (power of two)
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) wq_gemm_kernel(const __grid_constant__ GemmParams p) {
    using L = Layout<NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarriers);  // kStages + 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kStages + 1);
    int* flags = reinterpret_cast<int*>(tmem_slot + 1);  // [0] ok, [1] last-CTA
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const uint32_t sbase = smem_u32(smem);

    if (tid == 0) {
        for (int s = 0; s <= kStages; ++s) mbar_init(smem_u32(&bars[s]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 1;
    }
    __syncwarp();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(L::kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t idesc = idesc_bf16(NT);

    const int64_t kq = p.k >> 2;  // code bytes per feature row
    int64_t it = 0;               // stages issued by this CTA (for the parities)
    uint32_t done_phase = 0;
    bool ok = true;
    const int64_t units = static_cast<int64_t>(p.nblocks) * p.splits;
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int nb = static_cast<int>(u / p.splits);
        const int ks = static_cast<int>(u % p.splits);
        const int64_t n0 = static_cast<int64_t>(nb) * kBlockN;
        const int64_t kb = ks * p.kseg;
        const int64_t ke = (kb + p.kseg) < p.k ? (kb + p.kseg) : p.k;
        const int64_t nsteps = (ke - kb) / kStageK;
        const int64_t row = n0 + tid;  // this thread's feature row
        const uint8_t* crow = p.codes + (row < p.n ? row : 0) * kq;
        for (int64_t step = 0; step < nsteps; ++step, ++it) {
            const int s = static_cast<int>(it % kStages);
            if (it >= kStages) {  // stage s free: its previous MMAs are done
                if (tid == 0 && !mbar_wait(smem_u32(&bars[s]), ((it / kStages) - 1) & 1))
                    flags[0] = 0;
                __syncthreads();
                if (!flags[0]) {
                    ok = false;
                    break;
                }
            }
            const int64_t k0 = kb + step * kStageK;
            const uint32_t a_base = sbase + s * L::kStage;
            const uint32_t b_base = a_base + 2 * L::kAtomA;
            // activations: NT rows x 256 B, rows >= M zero-filled
#pragma unroll
            for (int i = 0; i < NT / 8; ++i) {
                const int chunk = tid + i * kThreads;  // 0 .. NT*16-1
                const int r = chunk >> 4;              // batch row
                const int c = chunk & 15;              // 16-byte chunk of 256 B
                const int atom = c >> 3, cc = c & 7;
                const uint32_t dst = b_base + atom * L::kAtomB + r * 128 + ((cc ^ (r & 7)) << 4);
                const bool valid = r < p.m;
                const uint16_t* src = p.x + (valid ? r : 0) * p.k + k0 + c * 8;
                cp_async16_zfill(dst, src, valid ? 16u : 0u);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            // weights: this thread's row, 128 codes -> 16 chunks of 8 bf16
            uint4 w0 = make_uint4(0, 0, 0, 0), w1 = make_uint4(0, 0, 0, 0);
            if (row < p.n) {
                const uint4* src = reinterpret_cast<const uint4*>(crow + (k0 >> 2));
                w0 = __ldcs(src);
                w1 = __ldcs(src + 1);
            }
            const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int j = 0; j < 16; ++j) {  // chunk j: codes 8j .. 8j+7
                const uint32_t h16 = (words[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
                const uint4 v = decode8(h16, p.table_lo, p.table_hi);
                const int atom = j >> 3, cc = j & 7;
                const uint32_t dst = a_base + atom * L::kAtomA + tid * 128 + ((cc ^ (tid & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x),
                             "r"(v.y), "r"(v.z), "r"(v.w)
                             : "memory");
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kStageK / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;  // 16 bf16 of K inside the atom
                    const uint64_t ad = sw128_desc(a_base + (kk >> 2) * L::kAtomA + off);
                    const uint64_t bd = sw128_desc(b_base + (kk >> 2) * L::kAtomB + off);
                    mma_bf16(tmem, ad, bd, idesc, (step > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(smem_u32(&bars[s]));
            }
        }
        if (!ok) break;
        // all MMAs of this unit done
        if (tid == 0) {
            mma_commit(smem_u32(&bars[kStages]));
            if (!mbar_wait(smem_u32(&bars[kStages]), done_phase)) flags[0] = 0;
        }
        done_phase ^= 1;
        __syncthreads();
        if (!flags[0]) {
            ok = false;
            break;
        }
        tc_fence_after();
        // epilogue: thread = feature row, NT columns = batch rows
        const float scale = row < p.n ? __fmul_rn(__ldg(p.alpha + row), p.factor) : 0.0f;
#pragma unroll
        for (int c0 = 0; c0 < NT; c0 += 16) {
            float v[16];
            __syncwarp();
            tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int64_t m = c0 + j;
                if (m < p.m && row < p.n) {
                    if (p.splits == 1) {
                        p.y[m * p.n + row] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v[j], scale)));
                    } else {
                        p.partial[(static_cast<int64_t>(ks) * p.m + m) * p.n + row] = v[j];
                    }
                }
            }
        }
        tc_fence_before();
        if (p.splits > 1) {
            __threadfence();
            __syncthreads();
            if (tid == 0) flags[1] = atomicAdd(&p.counters[nb], 1) == p.splits - 1;
            __syncthreads();
            if (flags[1]) {  // last segment of this feature block: add in order
                __threadfence();
                if (row < p.n) {
                    for (int64_t m = 0; m < p.m; ++m) {
                        float acc = 0.0f;
                        for (int s2 = 0; s2 < p.splits; ++s2)
                            acc = __fadd_rn(acc, __ldcg(p.partial + (static_cast<int64_t>(s2) * p.m + m) *
                                                                      p.n + row));
                        p.y[m * p.n + row] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(acc, scale)));
                    }
                }
                if (tid == 0) p.counters[nb] = 0;
            }
        }
        __syncthreads();  // TMEM reads done before the next unit's MMAs
    }
    // teardown: drain this CTA's MMAs (bounded), free TMEM
    if (tid == 0 && it > 0) {
        mma_commit(smem_u32(&bars[kStages]));
        mbar_wait(smem_u32(&bars[kStages]), done_phase);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(L::kCols)
                     : "memory");
}

// ------------------------------------------------------------------- host


static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

struct Plan {
    int nt;
    int splits;
    int64_t kseg;
    int nblocks;
};

static Plan plan(int64_t m, int64_t n, int64_t k) {
    Plan pl;
    pl.nt = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : 128;
    pl.nblocks = static_cast<int>((n + kBlockN - 1) / kBlockN);
    const int64_t ksteps = k / kStageK;
    const int64_t target = 2 * static_cast<int64_t>(sm_count());
    int64_t s = (target + pl.nblocks - 1) / pl.nblocks;
    const int64_t max_s = ksteps / 4 > 0 ? ksteps / 4 : 1;  // >= 4 stages per segment
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    const int64_t steps_per = (ksteps + s - 1) / s;
    pl.kseg = steps_per * kStageK;
    pl.splits = static_cast<int>((k + pl.kseg - 1) / pl.kseg);
    return pl;
}

static bool table_of(int q, uint32_t& lo, uint32_t& hi, float& factor) {
    // numerator of the code c of 2-bit field f (c = 0, 1, -2, -1)
    const int cs[4] = {0, 1, -2, -1};
    int num[4];
    switch (q) {
        case PQ_SEQ2: for (int f = 0; f < 4; ++f) num[f] = 2 * cs[f] + 1; factor = 0.25f; break;
        case PQ_SEQ2_B: for (int f = 0; f < 4; ++f) num[f] = 2 * cs[f] + 1; factor = 1.0f / 3.0f; break;
        case PQ_TERNARY: for (int f = 0; f < 4; ++f) num[f] = 2 * cs[f]; factor = 1.0f / 3.0f; break;
        case PQ_LSQ2: case PQ_BINARY: for (int f = 0; f < 4; ++f) num[f] = cs[f]; factor = 1.0f; break;
        default: return false;
    }
    uint16_t e[4];
    for (int f = 0; f < 4; ++f) {  // small integers are exact in bf16
        const float v = static_cast<float>(num[f]);
        uint32_t u;
        __builtin_memcpy(&u, &v, 4);
        e[f] = static_cast<uint16_t>(u >> 16);
    }
    lo = (e[0] & 0xFFu) | ((e[1] & 0xFFu) << 8) | ((e[2] & 0xFFu) << 16) | ((e[3] & 0xFFu) << 24);
    hi = (e[0] >> 8) | ((e[1] >> 8) << 8) | ((e[2] >> 8) << 16) | (static_cast<uint32_t>(e[3] >> 8) << 24);
    return true;
}

template <int NT>
static cudaError_t launch(const GemmParams& p, int64_t units, cudaStream_t s) {
    using L = Layout<NT>;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(
            wq_gemm_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int64_t sms = sm_count();
    const unsigned grid = static_cast<unsigned>(units < sms ? units : sms);
    wq_gemm_kernel<NT><<<grid, kThreads, L::kBytes, s>>>(p);
    return cudaGetLastError();
}

}  // namespace pqg

using namespace pqg;

extern "C" {

int64_t pq_wq_gemm_workspace_bytes(pq_quant_t q, int64_t m, int64_t n, int64_t k) {
    uint32_t lo, hi;
    float f;
    if (!table_of(q, lo, hi, f) || m < 1 || m > 128 || n < 1 || k < kStageK || k % kStageK) return -1;
    const Plan pl = plan(m, n, k);
    if (pl.splits == 1) return 0;
    return static_cast<int64_t>(pl.splits) * m * n * 4 + static_cast<int64_t>(pl.nblocks) * 4 + 256;
}

pq_status_t pq_wq_gemm(pq_quant_t q, int64_t m, int64_t n, int64_t k, const uint16_t* x_bf16,
                       const uint8_t* packed, const float* alpha, uint16_t* y_bf16, void* workspace,
                       int64_t workspace_bytes, void* stream) {
    GemmParams p = {};
    if (!table_of(q, p.table_lo, p.table_hi, p.factor)) return PQ_ERR_UNSUPPORTED;
    if (m < 1 || m > 128 || n < 1 || k < kStageK || k % kStageK) return PQ_ERR_INVALID_ARG;
    if (!x_bf16 || !packed || !alpha || !y_bf16) return PQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) || (reinterpret_cast<uintptr_t>(packed) & 15) ||
        (reinterpret_cast<uintptr_t>(y_bf16) & 1))
        return PQ_ERR_MISALIGNED;
    const Plan pl = plan(m, n, k);
    const int64_t need = pq_wq_gemm_workspace_bytes(q, m, n, k);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    p.x = x_bf16;
    p.codes = packed;
    p.alpha = alpha;
    p.y = y_bf16;
    p.m = m;
    p.n = n;
    p.k = k;
    p.kseg = pl.kseg;
    p.splits = pl.splits;
    p.nblocks = pl.nblocks;
    if (pl.splits > 1) {
        if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
            return PQ_ERR_INVALID_ARG;
        p.partial = static_cast<float*>(workspace);
        p.counters = reinterpret_cast<int*>(static_cast<char*>(workspace) +
                                            static_cast<int64_t>(pl.splits) * m * n * 4);
        if (cudaMemsetAsync(p.counters, 0, static_cast<size_t>(pl.nblocks) * 4, s) != cudaSuccess)
            return PQ_ERR_CUDA;
    }
    const int64_t units = static_cast<int64_t>(pl.nblocks) * pl.splits;
    cudaError_t e;
    switch (pl.nt) {
        case 16: e = launch<16>(p, units, s); break;
        case 32: e = launch<32>(p, units, s); break;
        case 64: e = launch<64>(p, units, s); break;
        default: e = launch<128>(p, units, s); break;
    }
    return e == cudaSuccess ? PQ_OK : PQ_ERR_CUDA;
}

int pq_device_status(void) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    }
    return v;
}

}  // extern "C"

// ------------------------------------------------- no-alloc entry point
// Split-K scratch of pq_wq_gemm_noalloc: one fixed array per device, shared
// by every call on that device; its address is looked up once per device.
namespace pqg {
static __device__ __align__(256) unsigned char g_noalloc_scratch[PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES];
constexpr int kNoAllocDevices = 256;
static std::atomic<void*> g_noalloc_addr[kNoAllocDevices];
}  // namespace pqg

extern "C" pq_status_t pq_wq_gemm_noalloc(pq_quant_t q, int64_t m, int64_t n, int64_t k,
                                          const uint16_t* x_bf16, const uint8_t* packed,
                                          const float* alpha, uint16_t* y_bf16, void* stream) {
    uint32_t lo, hi;
    float factor;
    if (!table_of(q, lo, hi, factor)) return PQ_ERR_UNSUPPORTED;
    if (m < 1 || m > 128 || n < 1 || k < kStageK || k % kStageK || !x_bf16 || !packed || !alpha ||
        !y_bf16)
        return PQ_ERR_INVALID_ARG;
    if (pq_wq_gemm_workspace_bytes(q, m, n, k) > PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES)
        return PQ_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PQ_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocDevices) return PQ_ERR_UNSUPPORTED;
    void* scratch = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (!scratch) {
        if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch)
            return PQ_ERR_CUDA;
        g_noalloc_addr[dev].store(scratch, std::memory_order_release);
    }
    return pq_wq_gemm(q, m, n, k, x_bf16, packed, alpha, y_bf16, scratch,
                      PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES, stream);
}
