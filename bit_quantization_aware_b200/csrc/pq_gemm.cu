// Weight-only low-bit matmul on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
//   Y[m][n] = sum_k X[m][k] * level(code[n][k]) * alpha[n]
//
// X: bf16 [M, K] activations (M <= 128, a decode-sized batch); codes: the
// forward's packed 2-bit codes [N, K/4]; alpha: fp32 [N]; Y: bf16 [M, N].
//
// Decoding. Every 2-bit level is affine in the code's offset-binary field
// f' = f xor 2 (c = f' - 2): numerator = A f' + B with (A, B) = (2, -3) for
// SEQ2 and SEQ2_B (2c + 1), (2, -4) for ternary (2c), (1, -2) for LSQ2 and
// binary (c). So a weight is decoded to the bf16 value 1 + f'/4, built by
// placing f' in the top two mantissa bits of 1.0 (one shift and one
// three-input logic op per two weights), and the tensor cores accumulate
//   D[r][j] = sum_k x[j][k] (1 + f'/4) = Sx[j] + (1/4) sum_k x[j][k] f'
// in fp32, with Sx[j] = sum_k x[j][k]. A 128-row tile holds 127 weight rows
// and one row of ones, whose accumulator is Sx itself, so
//   Y = alpha * factor * (4A D + (B - 4A) Sx) = alpha * (P D + Q Sx).
// The two weights decoded together are the code word's fields j and j + 8
// (16 bits apart), so the K order inside every group of 16 is interleaved
// (j, j + 8); the activation tile is permuted the same way in shared memory.
//
// Integer mode (m <= 16; this 8-bit form serves rows longer than 2^20, the
// packed-fp4 form below all others). The 8-bit MMA kinds take K = 32 per
// instruction at the cost of a K = 16 bf16 one, so the weights are decoded
// instead to their offset-binary fields f' as unsigned bytes (one shift and
// one three-input logic op per four weights) and multiplied (kind::i8, s32
// accumulators) by the activations in fixed point: a pre-pass scales each
// activation row by
// 2^(29 - E), E = floor(log2 max|x|), rounds to integers and writes their four
// signed base-256 digits as four planes, so the tensor cores form the exact
// integer sums of digits times fields, combined in fp64 in the epilogue:
//   Y = alpha * factor * (A * sum x f' + B * Sx)
// with Sx from the row of ones as before. The decoded bytes of a word are
// fields (s, s + 4, s + 8, s + 12), so the K order inside every group of 16
// is a 4 x 4 transpose, which the pre-pass applies to the planes.
//
// Packed-fp4 mode (m <= 16, k <= 2^20). Block-scaled fp4 MMAs
// (kind::mxf4, every scale 1.0) take K = 64 per instruction at about the cost
// of a K = 32 8-bit one, so the same exact integer sums run at twice the K
// per MMA. The weights go in as f'/2 (the e2m1 nibbles 0, 0.5, 1, 1.5 are
// the field's two bits in the low half of a nibble: one mask and one xor per
// eight weights), the same fixed-point activations v = rint(x 2^(29 - E)) as
// ten planes of balanced base-9 digits in [-4, 4] (all exact e2m1 values;
// |v| < 2^30 < 9^10 / 2). Every product is a multiple of 1/2 and every
// partial sum stays below 2^23 in magnitude for k <= 2^20, so the fp32
// accumulators hold exact integers, and the epilogue forms
// sum_k v f' = sum_p 9^p (2 acc_p) exactly in int64: the same integers as
// the 8-bit form's, through the same formula. The decoded nibbles of a code
// word are its even fields, then its odd fields, so the K order inside every
// group of 16 is (0, 2, .., 14, 1, 3, .., 15), which the pre-pass applies to
// the planes.
//
// Operands. A (decoded weights) lives in TMEM (tcgen05.st from the decode
// warps; tcgen05.mma reads it there, with no shared-memory round trip);
// B (activations) arrives by TMA in the 128B-swizzled K-major layout the
// MMA reads; the codes arrive by TMA, 512 K (128 B) per row per chunk, in a
// ring several chunks deep so that enough bytes are in flight per SM.
//
// Work split. The (row block, code chunk) items are cut into equal
// contiguous ranges, one per CTA (stream-K); a range covers whole blocks and
// at most two partial blocks. A partial block's pieces go to a caller
// workspace and the last CTA to finish the block adds them in K order
// (deterministic).
//
// Roles (19 warps in the bf16 mode, 15 in the integer and fp4 modes): 8
// decode warps (TMEM lane quarter = warp % 4, K half = warp / 4), 4 epilogue
// warps, 4 activation permuters (bf16 mode only: in the fixed-point modes the
// planes arrive already in MMA order and the MMA issuer waits for each
// stage's activations itself, 6-9% faster than a decode warp holding the
// stage until they land, which was itself 7% faster than a permuter pass),
// one codes producer, one activation producer, one MMA issuer. The
// activation ring is deeper than the A ring and has its own barriers, so
// decoding never waits on it. Every mbarrier wait is bounded: on giving up the kernel
// records a device status and an abort flag that ends every role's loop,
// waits (bounded) for its own copies and MMAs in flight, frees its TMEM and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <stdint.h>

#include <atomic>
#include <mutex>

#include "pq.h"
#include "pq_launches.cuh"

namespace pqg {

constexpr int kFeat = 127;             // weight rows per tile; TMEM lane 127 = ones
constexpr int kStageK = 256;           // K per MMA stage: 128 TMEM columns of A, 16 MMAs
constexpr int kChunkK = 512;           // K per codes chunk: 128 B per row
constexpr int kMinK = 128;             // K granularity of the problem
constexpr int kDecWarps = 8;           // warps 0..7
constexpr int kEpiWarp0 = 8;           // warps 8..11
constexpr int kPermWarp0 = 12;         // warps 12..15
constexpr int kPermWarps = 4;
// The single-thread roles follow the permuters (bf16) or the epilogue
// (integer and fp4 modes, which have no permuters): 19 or 15 warps, so the
// fixed-point instances get 128 registers a thread instead of 96.
template <int MODE>
struct Roles {
    static constexpr bool kPerm = MODE == 0;  // kModeBF16
    static constexpr int kCodesWarp = kPerm ? 16 : 12, kXWarp = kCodesWarp + 1, kMmaWarp = kCodesWarp + 2;
    static constexpr int kThreads = (kCodesWarp + 3) * 32;
};
constexpr uint32_t kTmemCols = 512;
constexpr int kCodesSlotBytes = 16384;
constexpr uint32_t kCodesTx = kFeat * 128;
constexpr uint32_t kMaxSpins = 1u << 22;
constexpr uint32_t kOnes = 0x3F803F80u;  // two bf16 1.0
constexpr uint32_t kOnesF4 = 0x22222222u;  // eight e2m1 1.0
constexpr uint32_t kScaleOne = 0x7F7F7F7Fu;  // four ue8m0 1.0
constexpr int kF4Planes = 10;            // base-9 digit planes of 30-bit fixed point
constexpr int64_t kF4MaxK = int64_t{1} << 20;  // exact fp32 sums up to this k

// Arithmetic of a launch: bf16 (kind::f16, m > 16), integer (kind::i8) or
// packed fp4 (kind::mxf4) on the same fixed-point activations.
enum : int { kModeBF16 = 0, kModeI8 = 1, kModeF4 = 2 };

// nonzero after a bounded wait gave up (read by pq_device_status)
__device__ int g_status = 0;
// nonzero: every launch raises its abort flag at start, so its waits give up
// as if their cap had been reached (pq_debug_abort_waits; tests the path)
__device__ int g_force_abort = 0;

// One matrix of a launch: its tensor maps, outputs and place in the work list.
struct Problem {
    CUtensorMap tc;      // codes [n rows][k/4 bytes], boxes of 127 rows x 128 B
    CUtensorMap tx;      // activations [m rows][k], boxes of NT rows x 64 K
    const float* alpha;  // [n]
    uint16_t* y;         // [m, n] bf16
    int64_t n, k;
    int64_t nchunks;     // ceil(k / kChunkK)
    int64_t item0;       // its first (block, chunk) item in the launch's list
    int64_t block0;      // its first block counter
    const int* xexp;     // integer mode: per activation row, the exponent E of max|x|
};

// Shared by the matrices of a launch (same activation rows m).
struct GemmCommon {
    float* partial;      // [2 * grid, kFeat, m4] fp32 (partial blocks only)
    int* counters;       // [all blocks], zero on entry (partial blocks only)
    int64_t m, m4;       // activation rows; m rounded up to a multiple of 4
    int64_t items;       // items of all matrices
    int32_t grid, count;
    float P, Q;          // y = alpha * (P * D + Q * Sx)
    double P4, PQ;       // integer mode: y = alpha * (P4 * sum x f' + PQ * Sx)
};

template <int MAXP>
struct GemmParams {
    GemmCommon c;
    Problem prob[MAXP];
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
           (static_cast<uint32_t>(128 >> 4) << 24);
}

// Instruction descriptor, kind::i8: s32 accumulator, A unsigned 8-bit, B
// signed 8-bit, both K-major, M = 128, N = nt.
__host__ __device__ constexpr uint32_t idesc_i8(int nt) {
    return (2u << 4) | (1u << 10) | (static_cast<uint32_t>(nt >> 3) << 17) |
           (static_cast<uint32_t>(128 >> 4) << 24);
}

// Instruction descriptor, kind::mxf4 with 32-element scale blocks: e2m1 A
// and B, ue8m0 scales, both K-major, M = 128, N = nt, K = 64.
__host__ __device__ constexpr uint32_t idesc_mxf4(int nt) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nt >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(128 >> 4) << 24);
}

// D (TMEM) (+)= A (TMEM) * B (shared memory)^T; K = 16 (bf16), 32 (8-bit) or
// 64 (fp4; the A and B scale factors come from TMEM columns sf.. and
// sf + 8.., all of whose bytes are 1.0: the two block scales of an operand's
// row r sit in column base + r / 32, lane r % 32 of every lane quarter that
// reads them, so 32 such columns over all 128 lanes serve N up to 192).
template <int MODE>
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate, uint32_t sf) {
    if (MODE == kModeF4)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], [%1], %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(tmem_d),
            "r"(tmem_a), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sf), "r"(sf + 8u)
            : "memory");
    else if (MODE == kModeI8)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
            "r"(tmem_a), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
            "r"(tmem_a), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     mbar)
                 : "memory");
}

// NK MMAs over one stage, each reading 32 bytes of K per row (16 bf16,
// 32 8-bit or 64 fp4 values): A columns advance by 8, the B descriptor start
// address by 32 B inside a 128-B swizzle atom and by one atom (ATOM_B bytes)
// every 4 MMAs.
template <int NK, int ATOM_B, int MODE>
__device__ __forceinline__ void issue_stage(uint32_t d, uint32_t a, uint64_t b0, uint32_t idesc,
                                            uint32_t acc0, uint32_t sf) {
#pragma unroll
    for (int kk = 0; kk < NK; ++kk)
        mma_ts<MODE>(d, a + 8u * kk, b0 + static_cast<uint64_t>(((kk >> 2) * ATOM_B + (kk & 3) * 32) >> 4),
                     idesc, kk == 0 ? acc0 : 1u, sf);
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t mbar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for the phase of the given parity (one thread). Gives up
// early when another role raised the abort flag; raises it (and the device
// status) when the spin limit is reached.
// The loop is kept to the barrier try and a periodic abort check: other
// work in it (even a rarely executed load) measurably slowed the pipeline.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, volatile int* abort) {
    for (uint32_t i = 0; i < kMaxSpins; ++i) {
        if (mbar_try(mbar, parity)) return true;
        if ((i & 63u) == 63u && *abort) return false;
    }
    *abort = 1;
    atomicExch(&g_status, 1);
    return false;
}

// The same, taken by lane 0 for the whole warp (the result is warp-uniform,
// so the warp stays converged for the .sync.aligned tensor-memory ops).
__device__ __forceinline__ bool warp_wait(uint32_t mbar, uint32_t parity, volatile int* abort) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(mbar, parity, abort) ? 1 : 0;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Bounded wait that ignores the abort flag (draining on the way out).
__device__ __forceinline__ void mbar_drain(uint32_t mbar, uint32_t parity) {
    for (uint32_t i = 0; i < kMaxSpins; ++i)
        if (mbar_try(mbar, parity)) return;
    atomicExch(&g_status, 1);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t mbar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(x), "r"(y)
        : "memory");
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
__device__ __forceinline__ void epi_sync() {  // the 4 epilogue warps
    asm volatile("bar.sync 1, 128;" ::: "memory");
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

// 8 fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z),
                 "r"(w)
                 : "memory");
}

// Fields j and j + 8 of a code word (two's complement, first column in the
// lowest bits) as two bf16 values 1 + f'/4 (low half: field j), with
// f' = f xor 2: the field lands in mantissa bits 5-6 of 1.0 and its sign
// bit is flipped there.
// select(b, a ^ c, c) in one three-input logic op: where the mask b is set,
// a with the sign bits of c flipped; elsewhere the constant bits of c.
__device__ __forceinline__ uint32_t mask_flip_or(uint32_t a, uint32_t b_imm_mask, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b_imm_mask), "r"(c));
    return d;
}

template <int J>
__device__ __forceinline__ uint32_t pair_of(uint32_t w) {
    const uint32_t s = J < 3 ? (w << (5 - 2 * J)) : (w >> (2 * J - 5));
    return ((s & 0x00600060u) ^ 0x00400040u) | kOnes;
}

// Integer mode: the 16 fields of a code word as four words of 8-bit
// offset-binary values f' = f xor 2 in 0..3; output s holds fields s, s + 4,
// s + 8, s + 12 (one per byte), so the K order inside every group of 16 is
// the 4 x 4 transpose (position 4s + b holds field s + 4b).
__device__ __forceinline__ void decode_word_u8(uint32_t w, uint32_t* v) {
    v[0] = mask_flip_or(w, 0x03030303u, 0x02020202u);
    v[1] = mask_flip_or(w >> 2, 0x03030303u, 0x02020202u);
    v[2] = mask_flip_or(w >> 4, 0x03030303u, 0x02020202u);
    v[3] = mask_flip_or(w >> 6, 0x03030303u, 0x02020202u);
}

// fp4 mode: the 16 fields of a code word as two words of e2m1 nibbles f'/2
// (f' = f xor 2 in the nibble's low two bits: 0, 0.5, 1, 1.5): the even
// fields, then the odd ones (K order (0, 2, .., 14, 1, 3, .., 15)).
__device__ __forceinline__ void decode_word_f4(uint32_t w, uint32_t* v) {
    v[0] = mask_flip_or(w, 0x33333333u, 0x22222222u);
    v[1] = mask_flip_or(w >> 2, 0x33333333u, 0x22222222u);
}

__device__ __forceinline__ void decode_word(uint32_t w, uint32_t* v) {
    v[0] = pair_of<0>(w);
    v[1] = pair_of<1>(w);
    v[2] = pair_of<2>(w);
    v[3] = pair_of<3>(w);
    v[4] = pair_of<4>(w);
    v[5] = pair_of<5>(w);
    v[6] = pair_of<6>(w);
    v[7] = pair_of<7>(w);
}

// Position in a ring of N mbarrier-guarded slots: slot index and the parity
// of its current phase. A wait on parity (phase ^ 1) passes at once on a
// fresh barrier, so a producer's first round needs no special case.
template <int N>
struct Ring {
    uint32_t idx = 0, phase = 0;
    __device__ __forceinline__ void next() {
        if (++idx == N) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

// Bounded wait for the last min(issued, N) loads of a full-barrier ring.
template <int N>
__device__ __forceinline__ void drain_ring(uint32_t bar0, Ring<N> r, uint32_t issued) {
    const uint32_t n = issued < static_cast<uint32_t>(N) ? issued : static_cast<uint32_t>(N);
    for (uint32_t j = 0; j < n; ++j) {
        if (r.idx == 0) {
            r.idx = N;
            r.phase ^= 1u;
        }
        --r.idx;
        mbar_drain(bar0 + 8u * r.idx, r.phase);
    }
}

// One piece of a CTA's range: matrix pi, row block b, code chunks [c0, c1).
struct Piece {
    int pi;
    int64_t b, c0, c1;
};

// Items [s, e) of CTA g. The items of matrix p are item0 + b * nchunks + chunk.
__device__ __forceinline__ int64_t range_start(const GemmCommon& p, int64_t g) {
    return g * p.items / p.grid;
}

// Next piece of [s, e); cur is the matrix the walk is in (items only grow).
template <int MAXP>
__device__ __forceinline__ bool next_piece(const GemmParams<MAXP>& prm, int64_t& s, int64_t e,
                                           Piece& pc, int& cur) {
    if (s >= e) return false;
    while (cur + 1 < prm.c.count && s >= prm.prob[cur + 1].item0) ++cur;
    const Problem& pb = prm.prob[cur];
    const int64_t local = s - pb.item0;
    const int64_t b = local / pb.nchunks;
    const int64_t blk_end = pb.item0 + (b + 1) * pb.nchunks;
    const int64_t pe = e < blk_end ? e : blk_end;
    pc.pi = cur;
    pc.b = b;
    pc.c0 = local - b * pb.nchunks;
    pc.c1 = pe - pb.item0 - b * pb.nchunks;
    s = pe;
    return true;
}

// fp4 decoders: a walk over a CTA's stages (one 512-K code chunk each),
// keeping the current matrix's k (read once per piece).
struct StageCursor {
    int64_t s, e;
    int cur;
    Piece pc;
    int64_t c, k;
    bool valid;
    template <int MAXP>
    __device__ __forceinline__ void piece(const GemmParams<MAXP>& prm) {
        valid = next_piece(prm, s, e, pc, cur);
        if (valid) {
            c = pc.c0;
            k = prm.prob[pc.pi].k;
        }
    }
    template <int MAXP>
    __device__ __forceinline__ void start(const GemmParams<MAXP>& prm, int64_t rs, int64_t re) {
        s = rs;
        e = re;
        cur = 0;
        piece(prm);
    }
    template <int MAXP>
    __device__ __forceinline__ void next(const GemmParams<MAXP>& prm) {
        if (++c >= pc.c1) piece(prm);
    }
    // K of this chunk left from the start of this thread's half (<= 0: none)
    __device__ __forceinline__ int64_t rest(int half) const { return k - (c * kChunkK + 256 * half); }
};

// MMA stages of SK K each in code chunk c of a K-long row (the last chunk
// may be short).
template <int SK>
__device__ __forceinline__ int stages_of_chunk(int64_t k, int64_t c) {
    const int64_t rest = (k - c * kChunkK + SK - 1) / SK;
    return rest < kChunkK / SK ? static_cast<int>(rest) : kChunkK / SK;
}

// K of the stage starting at k0: SK, or less (a multiple of 128) for a short tail.
template <int SK>
__device__ __forceinline__ int stage_k(int64_t k, int64_t k0) {
    return k - k0 < SK ? static_cast<int>(k - k0) : SK;
}

// CTA whose range holds item i: the largest g with range_start(g) <= i.
__device__ __forceinline__ int64_t cta_of_item(const GemmCommon& p, int64_t i) {
    return ((i + 1) * p.grid + p.items - 1) / p.items - 1;
}

// Shared memory and TMEM of one instance. bf16: 256 K per stage (four
// 64-K activation atoms), A slots of 128 TMEM columns; integer mode: 512 K
// per stage (four 128-K atoms), 128 columns; fp4: 512 K per stage (two
// 256-K atoms), 64 columns, plus 32 columns of unit scale factors.
template <int NT, int MODE>
struct Layout {
    static constexpr bool F4 = MODE == kModeF4;
    static constexpr int kCodesSlots = F4 ? (NT == 80 ? 6 : 4) : NT == 16 ? 8 : NT == 32 ? 6 : 4;
    static constexpr int kASlots = F4 ? (NT == 80 ? 4 : 2) : NT == 128 ? 2 : 3;
    static constexpr uint32_t kASlotCols = F4 ? 64 : 128;
    static constexpr int kBSlots = F4 ? (NT == 80 ? 6 : 3) : NT <= 32 ? 6 : NT == 64 ? 4 : 2;
    static_assert(kBSlots <= 2 * kASlots, "the activation producer reads stage completions "
                                         "from the A ring; deeper B rings would alias phases");
    // two accumulators, 32-column aligned
    static constexpr uint32_t kAccStride = F4 ? (NT + 31) / 32 * 32 : NT == 128 ? 128 : 64;
    static constexpr uint32_t kACol0 = 2 * kAccStride;
    static constexpr uint32_t kSfCol = kACol0 + kASlotCols * kASlots;  // fp4 only
    static constexpr int kAtomB = NT * 128;             // NT rows x 128 B
    static constexpr int kBSlot = (F4 ? 2 : 4) * kAtomB;
    static constexpr int kCodesOff = 0;
    static constexpr int kBOff = kCodesSlots * kCodesSlotBytes;
    static constexpr int kBarOff = kBOff + kBSlots * kBSlot;
    // cfull, cempty [codes slots]; xfull [B slots]; afull, aempty [A
    // slots]; accfull, accempty [2]; drain
    static constexpr int kNumBars = 2 * kCodesSlots + kBSlots + 2 * kASlots + 4 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort, last, ok
    static constexpr int kSxOff = kMiscOff + 16;              // 128 floats
    static constexpr int kBytes = kSxOff + 128 * 4 + 1024;    // + alignment slack
    static_assert(kSfCol + (F4 ? 32 : 0) <= kTmemCols, "TMEM columns");
};

// Integer mode: the four digit-plane accumulators of one activation row,
// sum_p acc_p * 256^p, as an exact double (|value| < 2^47).
__device__ __forceinline__ double planes_value(const float* v) {
    const long long t = static_cast<long long>(__float_as_int(v[0])) +
                        static_cast<long long>(__float_as_int(v[1])) * 256 +
                        static_cast<long long>(__float_as_int(v[2])) * 65536 +
                        static_cast<long long>(__float_as_int(v[3])) * 16777216;
    return static_cast<double>(t);
}

// fp4 mode: 2 sum_p 9^p acc_p for the MP activation rows of this thread's
// TMEM lane (plane p of row j in column d + p MP + j). Each accumulator is a
// multiple of 1/2 below 2^23 in magnitude (an exact fp32 value), so twice it
// converts exactly, and the int64 sum (< 2^52) is exact.
template <int MP>
__device__ __forceinline__ void f4_plane_sums(uint32_t d, long long (&s2)[MP]) {
#pragma unroll
    for (int j = 0; j < MP; ++j) s2[j] = 0;
    long long w = 1;
#pragma unroll
    for (int pl = 0; pl < kF4Planes; ++pl) {
        float v[MP];
        if constexpr (MP == 16)
            tmem_ld16(d + 16u * pl, v);
        else
            tmem_ld8(d + 8u * pl, v);
#pragma unroll
        for (int j = 0; j < MP; ++j) s2[j] += w * static_cast<long long>(__float2int_rn(2.0f * v[j]));
        w *= 9;
    }
}

// 2^e as a double, for e in [-1022, 1023].
__device__ __forceinline__ double exp2_int(int e) {
    return __longlong_as_double(static_cast<long long>(e + 1023) << 52);
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                       __fadd_rn(a.w, b.w));
}

// MODE kModeI8: the integer mode (kind::i8; A = offset-binary fields as u8,
// B = the activations' signed base-256 digit planes, NT = 4 x activation
// rows), 512 K per stage; kModeF4: the packed-fp4 mode (kind::mxf4; A =
// f'/2 nibbles, B = ten base-9 digit planes of 8 or 16 rows each, NT = 80 or
// 160), 512 K per stage; kModeBF16 (kind::f16), 256 K per stage.
template <int NT, int MAXP, int MODE>
__global__ void __launch_bounds__(Roles<MODE>::kThreads, 1)
    wq_gemm_kernel(const __grid_constant__ GemmParams<MAXP> prm) {
    using L = Layout<NT, MODE>;
    constexpr int kCodesWarp = Roles<MODE>::kCodesWarp, kXWarp = Roles<MODE>::kXWarp,
                  kMmaWarp = Roles<MODE>::kMmaWarp;
    constexpr bool I8 = MODE == kModeI8, F4 = MODE == kModeF4;
    constexpr bool INT = MODE != kModeBF16;          // fixed-point activations, exact sums
    constexpr int SK = INT ? 2 * kStageK : kStageK;  // K per stage
    constexpr int KB = F4 ? 256 : I8 ? 128 : 64;     // K per 128-B activation box
    const GemmCommon& p = prm.c;
    constexpr int SC = L::kCodesSlots, SA = L::kASlots, SB = L::kBSlots;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
    const uint32_t sbase = smem_u32(smem);
    const uint32_t b_cfull = sbase + L::kBarOff, b_cempty = b_cfull + 8u * SC;
    const uint32_t b_xfull = b_cempty + 8u * SC, b_afull = b_xfull + 8u * SB;
    const uint32_t b_aempty = b_afull + 8u * SA, b_accfull = b_aempty + 8u * SA;
    const uint32_t b_accempty = b_accfull + 16u, b_drain = b_accempty + 16u;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    volatile int* epi_ok = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 12);
    float* sx = reinterpret_cast<float*>(smem + L::kSxOff);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < SC; ++s) {
            mbar_init(b_cfull + 8u * s, 1);
            mbar_init(b_cempty + 8u * s, kDecWarps);
        }
        for (int s = 0; s < SB; ++s) mbar_init(b_xfull + 8u * s, 1);
        for (int s = 0; s < SA; ++s) {
            // integer and fp4 modes: the decoders alone (the issuer waits
            // for the stage's activations itself); bf16: decoders and permuters
            mbar_init(b_afull + 8u * s, INT ? kDecWarps : kDecWarps + kPermWarps);
            mbar_init(b_aempty + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(b_accfull + 8u * b, 1);
            mbar_init(b_accempty + 8u * b, 4);
        }
        mbar_init(b_drain, 1);
        const int forced = *static_cast<volatile int*>(&g_force_abort);
        *abort = forced;
        if (forced) atomicExch(&g_status, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid == kCodesWarp * 32) {
        for (int i = 0; i < prm.c.count && i < 4; ++i) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&prm.prob[i].tc))
                         : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&prm.prob[i].tx))
                         : "memory");
        }
    }
    __syncwarp();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if constexpr (F4) {
        // the unit scale factors every fp4 MMA reads
        if (warp < 4) {
            uint32_t one[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) one[j] = kScaleOne;
            tmem_st32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + L::kSfCol, one);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    const int64_t rs = range_start(p, blockIdx.x), re = range_start(p, blockIdx.x + 1);

    if (warp == kCodesWarp) {
        // ---------------------------------------------- codes producer
        if (lane == 0) {
            Ring<SC> cr;
            uint32_t issued = 0;
            int64_t s = rs;
            Piece pc;
            int cur = 0;
            bool ok = true;
            while (ok && next_piece(prm, s, re, pc, cur)) {
                const CUtensorMap* tc = &prm.prob[pc.pi].tc;
                for (int64_t c = pc.c0; c < pc.c1; ++c) {
                    if (!mbar_wait(b_cempty + 8u * cr.idx, cr.phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(b_cfull + 8u * cr.idx, kCodesTx);
                    tma_load_2d(sbase + L::kCodesOff + cr.idx * kCodesSlotBytes, tc,
                                b_cfull + 8u * cr.idx, static_cast<int32_t>(c * (kChunkK / 4)),
                                static_cast<int32_t>(pc.b * kFeat));
                    cr.next();
                    ++issued;
                }
            }
            // the loads still in flight land before the CTA may exit
            drain_ring(b_cfull, cr, issued);
        }
    } else if (warp == kXWarp) {
        // ---------------------------------------- activation producer
        if (lane == 0) {
            Ring<SB> xr;
            Ring<SA> er;  // A-ring position of stage gs - SB
            uint32_t gs = 0;
            int64_t s = rs;
            Piece pc;
            int cur = 0;
            bool ok = true;
            while (ok && next_piece(prm, s, re, pc, cur)) {
                const int64_t pk = prm.prob[pc.pi].k;  // once per piece
                const CUtensorMap* tx = &prm.prob[pc.pi].tx;
                for (int64_t c = pc.c0; c < pc.c1 && ok; ++c) {
                    const int ns = stages_of_chunk<SK>(pk, c);
                    for (int i = 0; i < ns; ++i, ++gs) {
                        if (gs >= static_cast<uint32_t>(SB)) {  // B slot free: stage gs - SB done
                            if (!mbar_wait(b_aempty + 8u * er.idx, er.phase, abort)) {
                                ok = false;
                                break;
                            }
                            er.next();
                        }
                        const int64_t k0 = c * kChunkK + i * SK;
                        const int boxes = (stage_k<SK>(pk, k0) + KB - 1) / KB;
                        const uint32_t dst = sbase + L::kBOff + xr.idx * L::kBSlot;
                        mbar_expect_tx(b_xfull + 8u * xr.idx, static_cast<uint32_t>(boxes * NT * 128));
                        for (int bx = 0; bx < boxes; ++bx)
                            tma_load_2d(dst + bx * L::kAtomB, tx, b_xfull + 8u * xr.idx,
                                        static_cast<int32_t>((k0 + KB * bx) / (F4 ? 2 : 1)), 0);
                        xr.next();
                    }
                }
            }
            drain_ring(b_xfull, xr, gs);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------- MMA issuer
        // The issuing thread blocks on every tcgen05.mma, so its loop keeps
        // bookkeeping to a few 32-bit operations between MMAs: a piece's
        // stage counts come from one read of the matrix's k (the launch's
        // parameters are too large for the constant cache, and the MMA asm's
        // memory clobbers would otherwise reload it on every stage).
        if (lane == 0) {
            constexpr uint32_t idesc = F4 ? idesc_mxf4(NT) : I8 ? idesc_i8(NT) : idesc_bf16(NT);
            const uint32_t sf = tmem + L::kSfCol;
            Ring<SA> ar;
            Ring<SB> br;
            Ring<2> accr;
            int64_t s = rs;
            Piece pc;
            int cur = 0;
            bool ok = true;
            while (ok && next_piece(prm, s, re, pc, cur)) {
                if (!mbar_wait(b_accempty + 8u * accr.idx, accr.phase ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + L::kAccStride * accr.idx;
                uint32_t acc0 = 0;
                // the piece's K range [c0 * 512, min(c1 * 512, k)): whole
                // stages, then at most one short one (k is a multiple of 128)
                const int64_t pk = prm.prob[pc.pi].k;
                const int64_t kspan = (pc.c1 * kChunkK < pk ? pc.c1 * kChunkK : pk) - pc.c0 * kChunkK;
                const int nfull = static_cast<int>(kspan / SK);
                const int tail_k = static_cast<int>(kspan % SK);
                for (int i = 0; i <= nfull; ++i) {
                    if (i == nfull && tail_k == 0) break;
                    if (!mbar_wait(b_afull + 8u * ar.idx, ar.phase, abort)) {
                        ok = false;
                        break;
                    }
                    // fixed point: the planes arrive in MMA order (no permuter
                    // pass), so the issuer waits for the stage's activations
                    // itself (a wait on a completed barrier costs it nothing)
                    if (INT && !mbar_wait(b_xfull + 8u * br.idx, br.phase, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = tmem + L::kACol0 + L::kASlotCols * ar.idx;
                    const uint64_t b0 = sw128_desc(sbase + L::kBOff + br.idx * L::kBSlot);
                    if (i < nfull)
                        issue_stage<F4 ? 8 : 16, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                    else if constexpr (F4) {  // 64 K per MMA
                        if (tail_k == 128)
                            issue_stage<2, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                        else if (tail_k == 256)
                            issue_stage<4, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                        else
                            issue_stage<6, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                    } else if (!I8 || tail_k == 256)
                        issue_stage<8, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                    else if (tail_k == 128)
                        issue_stage<4, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                    else
                        issue_stage<12, L::kAtomB, MODE>(d, a, b0, idesc, acc0, sf);
                    acc0 = 1;
                    mma_commit(b_aempty + 8u * ar.idx);
                    ar.next();
                    br.next();
                }
                if (!ok) break;
                mma_commit(b_accfull + 8u * accr.idx);
                accr.next();
            }
            // every MMA issued by this thread completes before TMEM is freed
            mma_commit(b_drain);
            mbar_drain(b_drain, 0);
        }
    } else if (F4 && warp < kDecWarps) {
        // ----------------------------------------------- fp4 decoders
        // Software-pipelined: each thread decodes its row's 64 code bytes of
        // a stage (256 K) to 32 words of nibbles and releases the codes
        // slot, issues the next stage's code loads, and only then waits for
        // the stage's A slot and stores the nibbles, so the shared-memory
        // load latency overlaps that wait (measured 3-5% faster than
        // loading after the store).
        const int quarter = warp & 3, half = warp >> 2;
        const int r = quarter * 32 + lane;  // TMEM lane = A row
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        Ring<SC> cr;
        Ring<SA> ar;
        StageCursor qc;
        qc.start(prm, rs, re);
        bool ok = qc.valid;
        uint4 w[4];
        auto load = [&](void) {
            const uint32_t crow = sbase + L::kCodesOff + cr.idx * kCodesSlotBytes + r * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) w[q] = lds128(crow + (((4 * half + q) ^ (r & 7)) << 4));
        };
        if (ok) {
            ok = warp_wait(b_cfull + 8u * cr.idx, cr.phase, abort);
            if (ok) load();
        }
        while (ok && qc.valid) {
            const bool mine = qc.rest(half) > 0;
            uint32_t v[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                decode_word_f4(w[q].x, v + 8 * q);
                decode_word_f4(w[q].y, v + 8 * q + 2);
                decode_word_f4(w[q].z, v + 8 * q + 4);
                decode_word_f4(w[q].w, v + 8 * q + 6);
            }
            if (r == kFeat) {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = kOnesF4;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b_cempty + 8u * cr.idx);
            cr.next();
            qc.next(prm);
            if (qc.valid) {
                if (!warp_wait(b_cfull + 8u * cr.idx, cr.phase, abort)) {
                    ok = false;
                    break;
                }
                load();
            }
            if (!warp_wait(b_aempty + 8u * ar.idx, ar.phase ^ 1u, abort)) {
                ok = false;
                break;
            }
            if (mine) {
                tc_fence_after();
                tmem_st32(tmem + lane_addr + L::kACol0 + L::kASlotCols * ar.idx + 32u * half, v);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b_afull + 8u * ar.idx);
            ar.next();
        }
    } else if (warp < kDecWarps) {
        // ------------------------------------------------------ decoders
        const int quarter = warp & 3, half = warp >> 2;
        const int r = quarter * 32 + lane;  // TMEM lane = A row
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        Ring<SC> cr;
        Ring<SA> ar;
        int64_t s = rs;
        Piece pc;
        int cur = 0;
        bool ok = true;
        while (ok && next_piece(prm, s, re, pc, cur)) {
            const int64_t pk = prm.prob[pc.pi].k;  // once per piece
            for (int64_t c = pc.c0; c < pc.c1 && ok; ++c) {
                if (!warp_wait(b_cfull + 8u * cr.idx, cr.phase, abort)) {
                    ok = false;
                    break;
                }
                const uint32_t crow = sbase + L::kCodesOff + cr.idx * kCodesSlotBytes + r * 128;
                const int ns = stages_of_chunk<SK>(pk, c);
                for (int i = 0; i < ns; ++i) {
                    // this warp's half of the stage exists unless the stage is a short tail
                    const bool mine = stage_k<SK>(pk, c * kChunkK + i * SK) > SK / 2 * half;
                    // bf16: 128 K of this row (32 code bytes) -> 64 TMEM columns;
                    // integer mode: 256 K (64 code bytes) -> 64 TMEM columns
                    const int ch = INT ? 4 * half : 4 * i + 2 * half;
                    uint32_t v[32], v2[32];
                    uint4 c2 = make_uint4(0, 0, 0, 0), c3 = c2;
                    if (I8 && mine) {
                        // the first half decoded before the wait; the rest after the first store
                        const uint4 c0 = lds128(crow + ((ch ^ (r & 7)) << 4));
                        const uint4 c1 = lds128(crow + (((ch + 1) ^ (r & 7)) << 4));
                        c2 = lds128(crow + (((ch + 2) ^ (r & 7)) << 4));
                        c3 = lds128(crow + (((ch + 3) ^ (r & 7)) << 4));
                        decode_word_u8(c0.x, v);
                        decode_word_u8(c0.y, v + 4);
                        decode_word_u8(c0.z, v + 8);
                        decode_word_u8(c0.w, v + 12);
                        decode_word_u8(c1.x, v + 16);
                        decode_word_u8(c1.y, v + 20);
                        decode_word_u8(c1.z, v + 24);
                        decode_word_u8(c1.w, v + 28);
                        if (r == kFeat) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = 0x01010101u;
                        }
                    } else if (!INT && mine) {
                        // decode the whole stage before waiting for its slot
                        const uint4 c0 = lds128(crow + ((ch ^ (r & 7)) << 4));
                        const uint4 c1 = lds128(crow + (((ch + 1) ^ (r & 7)) << 4));
                        decode_word(c0.x, v);
                        decode_word(c0.y, v + 8);
                        decode_word(c0.z, v + 16);
                        decode_word(c0.w, v + 24);
                        decode_word(c1.x, v2);
                        decode_word(c1.y, v2 + 8);
                        decode_word(c1.z, v2 + 16);
                        decode_word(c1.w, v2 + 24);
                        if (r == kFeat) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = v2[j] = kOnes;
                        }
                    }
                    if (!warp_wait(b_aempty + 8u * ar.idx, ar.phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    if (mine) {
                        tc_fence_after();
                        const uint32_t col = tmem + lane_addr + L::kACol0 + L::kASlotCols * ar.idx + 64u * half;
                        tmem_st32(col, v);
                        if (I8) {
                            decode_word_u8(c2.x, v2);
                            decode_word_u8(c2.y, v2 + 4);
                            decode_word_u8(c2.z, v2 + 8);
                            decode_word_u8(c2.w, v2 + 12);
                            decode_word_u8(c3.x, v2 + 16);
                            decode_word_u8(c3.y, v2 + 20);
                            decode_word_u8(c3.z, v2 + 24);
                            decode_word_u8(c3.w, v2 + 28);
                            if (r == kFeat) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) v2[j] = 0x01010101u;
                            }
                        }
                        tmem_st32(col + 32u, v2);
                        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                        tc_fence_before();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_afull + 8u * ar.idx);
                    ar.next();
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(b_cempty + 8u * cr.idx);
                cr.next();
            }
        }
    } else if (!INT && warp >= kPermWarp0 && warp < kPermWarp0 + kPermWarps) {
        // ------------------- activation permuters: each group of 16 K -> (j, j + 8)
        // (bf16 mode only: the integer mode's digit planes arrive in MMA order)
        const int ptid = tid - kPermWarp0 * 32;
        Ring<SB> br;
        Ring<SA> ar;
        int64_t s = rs;
        Piece pc;
        int cur = 0;
        bool ok = true;
        while (ok && next_piece(prm, s, re, pc, cur)) {
            const int64_t pk = prm.prob[pc.pi].k;  // once per piece
            for (int64_t c = pc.c0; c < pc.c1 && ok; ++c) {
                const int ns = stages_of_chunk<SK>(pk, c);
                for (int i = 0; i < ns; ++i) {
                    if (!warp_wait(b_xfull + 8u * br.idx, br.phase, abort)) {
                        ok = false;
                        break;
                    }
                    // the integer mode's digit planes arrive already in MMA order
                    const int groups = INT ? 0 : stage_k<SK>(pk, c * kChunkK + i * SK) / 16;
                    const uint32_t bslot = sbase + L::kBOff + br.idx * L::kBSlot;
                    for (int it = ptid; it < NT * groups; it += kPermWarps * 32) {
                        const int bro = it % NT, g = it / NT;
                        const int ch = 2 * (g & 3);
                        const uint32_t rowa = bslot + (g >> 2) * L::kAtomB + bro * 128;
                        const uint32_t a0 = rowa + ((ch ^ (bro & 7)) << 4);
                        const uint32_t a1 = rowa + (((ch + 1) ^ (bro & 7)) << 4);
                        const uint4 A = lds128(a0), B = lds128(a1);
                        sts128(a0, __byte_perm(A.x, B.x, 0x5410), __byte_perm(A.x, B.x, 0x7632),
                               __byte_perm(A.y, B.y, 0x5410), __byte_perm(A.y, B.y, 0x7632));
                        sts128(a1, __byte_perm(A.z, B.z, 0x5410), __byte_perm(A.z, B.z, 0x7632),
                               __byte_perm(A.w, B.w, 0x5410), __byte_perm(A.w, B.w, 0x7632));
                    }
                    fence_async_smem();
                    // arrive only once this A-ring phase is the one for this stage
                    if (!warp_wait(b_aempty + 8u * ar.idx, ar.phase ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_afull + 8u * ar.idx);
                    ar.next();
                    br.next();
                }
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        // ------------------------------------------------------ epilogue
        const int e = warp - kEpiWarp0;
        const int r = e * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(e * 32) << 16;
        const int epi_leader = kEpiWarp0 * 32;
        Ring<2> accr;
        int64_t s = rs;
        Piece pc;
        int cur = 0;
        while (next_piece(prm, s, re, pc, cur)) {
            const uint32_t ab = accr.idx;
            // one thread waits; all four warps take the same branch
            if (tid == epi_leader)
                *epi_ok = mbar_wait(b_accfull + 8u * ab, accr.phase, abort) ? 1 : 0;
            epi_sync();
            if (!*epi_ok) break;
            tc_fence_after();
            const uint32_t d = tmem + lane_addr + L::kAccStride * ab;
            constexpr int MP = NT / kF4Planes;  // fp4: activation rows per plane
            // pass 1: Sx (TMEM lane 127) to shared memory, read by the one
            // warp whose lanes hold it (fp4: the ones row's A is 1.0, so its
            // plane sums are sum v itself, half of 2 sum_p 9^p acc_p)
            if constexpr (F4) {
                if (e == kFeat / 32) {
                    long long s2[MP];
                    f4_plane_sums<MP>(d, s2);
                    if (r == kFeat) {
#pragma unroll
                        for (int j = 0; j < MP; ++j)
                            reinterpret_cast<double*>(sx)[j] = 0.5 * static_cast<double>(s2[j]);
                    }
                }
            }
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
                if (F4 || e != kFeat / 32) break;
                float v[16];
                __syncwarp();
                tmem_ld16(d + c0, v);
                if (r == kFeat) {
                    if (I8) {
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            reinterpret_cast<double*>(sx)[c0 / 4 + jj] = planes_value(v + 4 * jj);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) sx[c0 + j] = v[j];
                    }
                }
            }
            epi_sync();
            const Problem& pb = prm.prob[pc.pi];
            const bool full = pc.c0 == 0 && pc.c1 == pb.nchunks;
            const int64_t feat = pc.b * kFeat + r;
            const bool valid_row = r < kFeat && feat < pb.n;
            const float alpha = valid_row ? __ldg(pb.alpha + feat) : 0.0f;
            // workspace row of a partial piece: slot 0 if it opens this CTA's range
            const int wslot = (pb.item0 + pc.b * pb.nchunks + pc.c0 == rs) ? 0 : 1;
            float* prow = full ? nullptr
                               : p.partial + ((static_cast<int64_t>(blockIdx.x) * 2 + wslot) * kFeat + r) * p.m4;
            if constexpr (F4) {
                // weight row r: sum_k v f' = 2 sum_p 9^p acc_p; x = v 2^(E - 29)
                long long s2[MP];
                __syncwarp();
                f4_plane_sums<MP>(d, s2);
                // the accumulator is read: hand it back before the arithmetic
                // and the stores
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_accempty + 8u * ab);
                float o[MP];
#pragma unroll
                for (int j = 0; j < MP; ++j) {
                    const double scale = j < p.m ? exp2_int(__ldg(pb.xexp + j) - 29) : 0.0;
                    o[j] = static_cast<float>(
                        (p.P4 * static_cast<double>(s2[j]) + p.PQ * reinterpret_cast<const double*>(sx)[j]) * scale);
                }
                if (valid_row) {
                    if (full) {
#pragma unroll
                        for (int j = 0; j < MP; ++j)
                            if (j < p.m)
                                pb.y[j * pb.n + feat] = __bfloat16_as_ushort(__float2bfloat16_rn(alpha * o[j]));
                    } else {
#pragma unroll
                        for (int j4 = 0; j4 < MP; j4 += 4)
                            if (j4 < p.m4)
                                *reinterpret_cast<float4*>(prow + j4) =
                                    make_float4(o[j4], o[j4 + 1], o[j4 + 2], o[j4 + 3]);
                    }
                }
            }
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
                if (F4) break;
                float v[16];
                __syncwarp();
                tmem_ld16(d + c0, v);
                if constexpr (I8) {
                    // columns 4j .. 4j + 3 are activation row j's digit planes;
                    // x = digits * 2^(E - 29)
                    float o[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = c0 / 4 + jj;
                        const double scale = j < p.m ? exp2_int(__ldg(pb.xexp + j) - 29) : 0.0;
                        o[jj] = static_cast<float>(
                            (p.P4 * planes_value(v + 4 * jj) + p.PQ * reinterpret_cast<const double*>(sx)[j]) * scale);
                    }
                    if (!valid_row) continue;
                    if (full) {
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            if (c0 / 4 + jj < p.m)
                                pb.y[(c0 / 4 + jj) * pb.n + feat] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(alpha * o[jj]));
                    } else if (c0 / 4 < p.m4) {
                        *reinterpret_cast<float4*>(prow + c0 / 4) = make_float4(o[0], o[1], o[2], o[3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = fmaf(p.P, v[j], p.Q * sx[c0 + j]);
                    if (!valid_row) continue;
                    if (full) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (c0 + j < p.m)
                                pb.y[(c0 + j) * pb.n + feat] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(alpha * v[j]));
                    } else {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            if (c0 + 4 * q4 < p.m4)
                                *reinterpret_cast<float4*>(prow + c0 + 4 * q4) = make_float4(
                                    v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                    }
                }
            }
            if (!F4) {  // (fp4: handed back right after its TMEM reads)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_accempty + 8u * ab);
            }
            if (!full) {
                // the last of the block's pieces to finish adds them in K order
                __threadfence();
                epi_sync();
                const int64_t i0 = pb.item0 + pc.b * pb.nchunks, i1 = i0 + pb.nchunks - 1;
                const int64_t g0 = cta_of_item(p, i0), g1 = cta_of_item(p, i1);
                if (tid == epi_leader)
                    *last_flag = atomicAdd(p.counters + pb.block0 + pc.b, 1) == static_cast<int>(g1 - g0);
                epi_sync();
                if (*last_flag) {
                    __threadfence();
                    if (valid_row) {
                        // CTA g0's piece opens its range iff the range starts at i0
                        const int slot0 = range_start(p, g0) >= i0 ? 0 : 1;
                        for (int64_t m0 = 0; m0 < p.m4; m0 += 16) {
                            float4 acc[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                            for (int64_t g = g0; g <= g1; ++g) {
                                const int sl = g == g0 ? slot0 : 0;
                                const float4* src = reinterpret_cast<const float4*>(
                                    p.partial + ((g * 2 + sl) * kFeat + r) * p.m4 + m0);
                                float4 t[4];
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    if (m0 + 4 * q < p.m4) t[q] = __ldcg(src + q);
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    if (m0 + 4 * q < p.m4) acc[q] = add4(acc[q], t[q]);
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float a4[4] = {acc[q].x, acc[q].y, acc[q].z, acc[q].w};
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const int64_t mr = m0 + 4 * q + j;
                                    if (mr < p.m)
                                        pb.y[mr * pb.n + feat] =
                                            __bfloat16_as_ushort(__float2bfloat16_rn(alpha * a4[j]));
                                }
                            }
                        }
                    }
                    if (tid == epi_leader) p.counters[pb.block0 + pc.b] = 0;
                }
            }
            epi_sync();  // sx, last_flag and epi_ok are reused by the next piece
            accr.next();
        }
    }

    // teardown: every role is done (or gave up); free TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

// Sixteen consecutive activations (bf16 pairs hw[0..7]) as the integer
// mode's four signed base-256 digit words per plane: v = rint(x * 2^(29-E))
// (ties to even; the product is exact in fp64),
// v = d0 + 256 d1 + 65536 d2 + 2^24 d3, digits in [-128, 127]; in plane p,
// byte position 4s + b holds the digit of element s + 4b (the decoded
// weights' K order).
__device__ __forceinline__ void digits16(const uint32_t (&hw)[8], int E, uint32_t (&pw)[4][4]) {
    const double sc = exp2_int(29 - E);
#pragma unroll
    for (int pp = 0; pp < 4; ++pp)
#pragma unroll
        for (int q = 0; q < 4; ++q) pw[pp][q] = 0;
#pragma unroll
    for (int f = 0; f < 16; ++f) {
        const uint32_t bits = (f & 1) ? (hw[f >> 1] & 0xFFFF0000u) : (hw[f >> 1] << 16);
        int v = __double2int_rn(static_cast<double>(__uint_as_float(bits)) * sc);
        const int pos = 4 * (f & 3) + (f >> 2);
#pragma unroll
        for (int pp = 0; pp < 3; ++pp) {
            const int dgt = ((v + 128) & 255) - 128;
            v = (v - dgt) >> 8;
            pw[pp][pos >> 2] |= static_cast<uint32_t>(dgt & 255) << (8 * (pos & 3));
        }
        pw[3][pos >> 2] |= static_cast<uint32_t>(v & 255) << (8 * (pos & 3));
    }
}

// fp4 mode: sixteen consecutive activations as the ten balanced base-9
// digit planes of the same fixed point v = rint(x * 2^(29-E)): v = sum_p
// 9^p d_p, d_p in [-4, 4] (|v| < 2^30 < 9^10 / 2), each digit as an e2m1
// nibble (0, 1, 2, 3, 4 = 0b0000, 0b0010, 0b0100, 0b0101, 0b0110; sign bit 3).
// Plane p's first word holds the even elements (element 2i in nibble i),
// its second word the odd ones: the decoded weights' K order.
__device__ __forceinline__ void digits16_f4(const uint32_t (&hw)[8], int E, uint32_t (&w0)[kF4Planes],
                                            uint32_t (&w1)[kF4Planes]) {
    const double sc = exp2_int(29 - E);
#pragma unroll
    for (int pp = 0; pp < kF4Planes; ++pp) w0[pp] = w1[pp] = 0;
#pragma unroll
    for (int f = 0; f < 16; ++f) {
        const uint32_t bits = (f & 1) ? (hw[f >> 1] & 0xFFFF0000u) : (hw[f >> 1] << 16);
        int v = __double2int_rn(static_cast<double>(__uint_as_float(bits)) * sc);
        const int sh = 4 * (f >> 1);
#pragma unroll
        for (int pp = 0; pp < kF4Planes; ++pp) {
            int dgt = v;  // the last plane takes what is left (|v| <= 3 there)
            if (pp + 1 < kF4Planes) {
                const int t = v + 4;
                const int q = (t >= 0 ? t : t - 8) / 9;  // floor(t / 9)
                dgt = t - 9 * q - 4;
                v = q;
            }
            const uint32_t mag = static_cast<uint32_t>(dgt < 0 ? -dgt : dgt);
            const uint32_t nib = (mag <= 2 ? 2 * mag : mag + 2) | (dgt < 0 ? 8u : 0u);
            if (f & 1)
                w1[pp] |= nib << sh;
            else
                w0[pp] |= nib << sh;
        }
    }
}

// floor(log2 |x|) of the largest magnitude among bf16 bit patterns given as
// their sign-cleared magnitude bits (0 for an all-zero row), subnormals included.
__device__ __forceinline__ int exponent_of_max(uint32_t mag_bits16) {
    const uint32_t b = mag_bits16 << 16;
    return b == 0 ? 0 : (b >> 23) ? static_cast<int>(b >> 23) - 127 : -118 - __clz(b);
}

// ------------------------------------------------- one activation row
// For m = 1 the tensor cores retire at most 2048 weights per ~46-cycle MMA
// per SM, far below what the codes' bandwidth allows, so a single row takes
// a CUDA-core path: each weight is decoded to the fp32 value 1 + f'/4 (one
// shift and one logic op) and multiplied into paired fp32 accumulators
// (two FMAs per instruction); the same affine identity gives
// y = alpha * (P * D + Q * Sx). x is held in shared memory as fp32 (each
// CTA converts it once per matrix and sums it in a fixed order; each 64-K
// chunk is padded so lanes reading consecutive chunks hit different banks); warps take
// tasks of 1, 2 or 4 rows from a per-matrix counter; lane l reads 16-byte chunks
// l, l + 32, ... of each row, so every load of a warp is 512 contiguous
// bytes; a fixed shuffle tree sums a row's lane partials (deterministic).
namespace pqv {

constexpr int kThreads = 512;
constexpr int64_t kMaxK = 32768;         // x as fp32 in shared memory: 136 KB padded
// 64 x values (16 float4) per chunk, padded to 17 float4: the 8 lanes of a
// quarter-warp read 8 consecutive chunks at the same offset, 68 floats apart,
// which falls in 8 different bank groups
constexpr int kChunkF4 = 17;

struct VecProblem {
    const uint16_t* x;   // [k] bf16
    const uint8_t* codes;  // [n, k/4]
    const float* alpha;  // [n]
    uint16_t* y;         // [n] bf16
    int64_t n, k;
    int* counter;        // task counter, zero on entry
    int32_t rows;        // rows per task: 1, 2 or 4 (about one task per warp or more)
};

template <int MAXP>
struct VecParams {
    int32_t count;
    float P, Q;
    double P4, PQ;       // integer kernel: y = alpha * (P4 * sum x f' + PQ * Sx)
    VecProblem prob[MAXP];
};

// Field j (0..7) of a code half-word h as the fp32 value 1 + f'/4 with
// f' = field xor 2: the field is moved to mantissa bits 21-22 by a multiply
// (an FMA-pipe instruction, which leaves the ALU pipe to the mask), then
// masked, its sign bit flipped, and the exponent of 1.0 set.
template <int J>
__device__ __forceinline__ float dec32(uint32_t h) {
    uint32_t s;
    asm("mul.lo.u32 %0, %1, %2;" : "=r"(s) : "r"(h), "n"(1u << (21 - 2 * J)));
    return __uint_as_float(mask_flip_or(s, 0x00600000u, 0x00400000u | 0x3F800000u));
}

// acc += x[0..15] * fields of w (x as 8 float2 pairs, paired FMAs); fields
// 8..15 are taken from the upper half after one shift, so every field needs
// only a left shift.
__device__ __forceinline__ float2 word_fma(uint32_t w, const float2* x, float2 acc) {
    const uint32_t hi = w >> 16;
    acc = __ffma2_rn(x[0], make_float2(dec32<0>(w), dec32<1>(w)), acc);
    acc = __ffma2_rn(x[1], make_float2(dec32<2>(w), dec32<3>(w)), acc);
    acc = __ffma2_rn(x[2], make_float2(dec32<4>(w), dec32<5>(w)), acc);
    acc = __ffma2_rn(x[3], make_float2(dec32<6>(w), dec32<7>(w)), acc);
    acc = __ffma2_rn(x[4], make_float2(dec32<0>(hi), dec32<1>(hi)), acc);
    acc = __ffma2_rn(x[5], make_float2(dec32<2>(hi), dec32<3>(hi)), acc);
    acc = __ffma2_rn(x[6], make_float2(dec32<4>(hi), dec32<5>(hi)), acc);
    acc = __ffma2_rn(x[7], make_float2(dec32<6>(hi), dec32<7>(hi)), acc);
    return acc;
}

// One task: rows task*R .. task*R + R - 1 of a matrix, whole K; lane l
// takes 16-byte code chunks l, l + 32, ...; x from shared memory is reused
// by the R rows. The loads of a lane's next chunk are issued before the
// current one is computed, so a load's latency overlaps a chunk of math.
template <int R>
__device__ __forceinline__ void row_task(const VecProblem& pb, int task, int64_t kq, int64_t nchunk,
                                         int lane, float P, float qsx, const float4* xs4) {
    const int64_t row0 = static_cast<int64_t>(task) * R;
    const uint8_t* rp[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t row = row0 + r < pb.n ? row0 + r : pb.n - 1;
        rp[r] = pb.codes + row * kq;
    }
    float2 acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = make_float2(0.0f, 0.0f);
    uint4 w[R];
    if (lane < nchunk) {
#pragma unroll
        for (int r = 0; r < R; ++r) w[r] = __ldcs(reinterpret_cast<const uint4*>(rp[r] + lane * 16));
    }
    for (int64_t c = lane; c < nchunk; c += 32) {
        uint4 wn[R];
        if (c + 32 < nchunk) {
#pragma unroll
            for (int r = 0; r < R; ++r) wn[r] = __ldcs(reinterpret_cast<const uint4*>(rp[r] + (c + 32) * 16));
        }
        const float4* xc = xs4 + c * kChunkF4;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float2 xv[8];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 f = xc[4 * q4 + u];
                xv[2 * u] = make_float2(f.x, f.y);
                xv[2 * u + 1] = make_float2(f.z, f.w);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t word = q4 == 0 ? w[r].x : q4 == 1 ? w[r].y : q4 == 2 ? w[r].z : w[r].w;
                acc[r] = word_fma(word, xv, acc[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) w[r] = wn[r];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float d = __fadd_rn(acc[r].x, acc[r].y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d = __fadd_rn(d, __shfl_xor_sync(0xFFFFFFFFu, d, o));
        const int64_t row = row0 + r;
        if (lane == r && row < pb.n)
            pb.y[row] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldg(pb.alpha + row) * fmaf(P, d, qsx)));
    }
}

template <int MAXP>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(const __grid_constant__ VecParams<MAXP> prm) {
    extern __shared__ float4 xs4[];  // 64-K chunk c at float4 c * kChunkF4 (padded)
    __shared__ float warp_sum[kThreads / 32];
    __shared__ float sx_sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int pi = 0; pi < prm.count; ++pi) {
        const VecProblem& pb = prm.prob[pi];
        const int64_t nq = pb.k / 4;  // float4 slots of x
        // x -> fp32 shared memory (chunks padded to 17 float4) and its sum
        float part = 0.0f;
        for (int64_t i = tid; i < nq; i += kThreads) {
            const uint2 h = __ldg(reinterpret_cast<const uint2*>(pb.x) + i);
            const float4 v = make_float4(__uint_as_float(h.x << 16), __uint_as_float(h.x & 0xFFFF0000u),
                                         __uint_as_float(h.y << 16), __uint_as_float(h.y & 0xFFFF0000u));
            xs4[(i >> 4) * kChunkF4 + (i & 15)] = v;
            part = __fadd_rn(__fadd_rn(part, v.x), __fadd_rn(v.y, __fadd_rn(v.z, v.w)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(0xFFFFFFFFu, part, o));
        if (lane == 0) warp_sum[warp] = part;
        __syncthreads();
        if (tid == 0) {
            float t = 0.0f;
            for (int w = 0; w < kThreads / 32; ++w) t = __fadd_rn(t, warp_sum[w]);
            sx_sh = t;
        }
        __syncthreads();
        const float sx = sx_sh;
        const float qsx = prm.Q * sx;
        const int64_t kq = pb.k / 4, nchunk = pb.k / 64;
        const int64_t ntasks = (pb.n + pb.rows - 1) / pb.rows;
        for (;;) {
            int task = 0;
            if (lane == 0) task = atomicAdd(pb.counter, 1);
            task = __shfl_sync(0xFFFFFFFFu, task, 0);
            if (task >= ntasks) break;
            if (pb.rows == 4) row_task<4>(pb, task, kq, nchunk, lane, prm.P, qsx, xs4);
            else if (pb.rows == 2) row_task<2>(pb, task, kq, nchunk, lane, prm.P, qsx, xs4);
            else row_task<1>(pb, task, kq, nchunk, lane, prm.P, qsx, xs4);
        }
        __syncthreads();  // the next matrix overwrites x
    }
}

// Integer one-row kernel: the integer mode's arithmetic on the CUDA cores.
// Each CTA turns x into four signed base-256 digit planes in shared memory
// (scale 2^(29 - E) from the row's largest magnitude, as in the pre-pass;
// chunk c of 64 K at c * 272 bytes, [word w][plane p] 16 bytes each, the K
// order transposed like the decoded fields) and sums their digits (Sx).
// A weight word gives four registers of u8 fields (one shift and one
// three-input op each), and dp4a multiplies each against the matching four
// digits of every plane: 23 instructions per 16 weights, exact int32 sums.
template <int R>
__device__ __forceinline__ void row_task_i8(const VecProblem& pb, int task, int64_t kq, int64_t nchunk,
                                            int lane, double P4, double PQ, double sxd, double scale,
                                            const uint4* xs4) {
    const int64_t row0 = static_cast<int64_t>(task) * R;
    const uint8_t* rp[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t row = row0 + r < pb.n ? row0 + r : pb.n - 1;
        rp[r] = pb.codes + row * kq;
    }
    int acc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) acc[r][pp] = 0;
    uint4 w[R];
    if (lane < nchunk) {
#pragma unroll
        for (int r = 0; r < R; ++r) w[r] = __ldcs(reinterpret_cast<const uint4*>(rp[r] + lane * 16));
    }
    for (int64_t c = lane; c < nchunk; c += 32) {
        uint4 wn[R];
        if (c + 32 < nchunk) {
#pragma unroll
            for (int r = 0; r < R; ++r) wn[r] = __ldcs(reinterpret_cast<const uint4*>(rp[r] + (c + 32) * 16));
        }
        const uint4* xc = xs4 + c * kChunkF4;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            uint4 xp[4];
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) xp[pp] = xc[4 * q4 + pp];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t word = q4 == 0 ? w[r].x : q4 == 1 ? w[r].y : q4 == 2 ? w[r].z : w[r].w;
                uint32_t o[4];
                decode_word_u8(word, o);
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    int a = acc[r][pp];
                    a = __dp4a(static_cast<int>(o[0]), static_cast<int>(xp[pp].x), a);
                    a = __dp4a(static_cast<int>(o[1]), static_cast<int>(xp[pp].y), a);
                    a = __dp4a(static_cast<int>(o[2]), static_cast<int>(xp[pp].z), a);
                    a = __dp4a(static_cast<int>(o[3]), static_cast<int>(xp[pp].w), a);
                    acc[r][pp] = a;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) w[r] = wn[r];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        long long t = 0;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            int a = acc[r][pp];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
            t += static_cast<long long>(a) * (1LL << (8 * pp));
        }
        const int64_t row = row0 + r;
        if (lane == r && row < pb.n) {
            const float v = static_cast<float>((P4 * static_cast<double>(t) + PQ * sxd) * scale);
            pb.y[row] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldg(pb.alpha + row) * v));
        }
    }
}

template <int MAXP>
__global__ void __launch_bounds__(kThreads, 1) gemv_i8_kernel(const __grid_constant__ VecParams<MAXP> prm) {
    extern __shared__ uint4 xq[];  // 64-K chunk c at uint4 c * kChunkF4: [word][plane]
    __shared__ uint32_t red_mb[kThreads / 32];
    __shared__ int red_s[kThreads / 32][4];
    __shared__ int e_sh;
    __shared__ double sx_sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int pi = 0; pi < prm.count; ++pi) {
        const VecProblem& pb = prm.prob[pi];
        // max |x| of the row
        uint32_t mb = 0;
        for (int64_t i = tid; i < pb.k / 8; i += kThreads) {
            const uint4 h = __ldg(reinterpret_cast<const uint4*>(pb.x) + i);
            const uint32_t a = __vmaxu2(__vmaxu2(h.x & 0x7FFF7FFFu, h.y & 0x7FFF7FFFu),
                                        __vmaxu2(h.z & 0x7FFF7FFFu, h.w & 0x7FFF7FFFu));
            mb = max(mb, max(a & 0xFFFFu, a >> 16));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
        if (lane == 0) red_mb[warp] = mb;
        __syncthreads();
        if (tid == 0) {
            uint32_t t = red_mb[0];
            for (int w = 1; w < kThreads / 32; ++w) t = max(t, red_mb[w]);
            e_sh = exponent_of_max(t);
        }
        __syncthreads();
        const int E = e_sh;
        // digit planes into shared memory, and the planes' digit sums
        int s4[4] = {0, 0, 0, 0};
        for (int64_t g = tid; g < pb.k / 16; g += kThreads) {
            const uint4 h0 = __ldg(reinterpret_cast<const uint4*>(pb.x + 16 * g));
            const uint4 h1 = __ldg(reinterpret_cast<const uint4*>(pb.x + 16 * g) + 1);
            const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            uint32_t pw[4][4];
            digits16(hw, E, pw);
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                xq[(g >> 2) * kChunkF4 + 4 * (g & 3) + pp] = make_uint4(pw[pp][0], pw[pp][1], pw[pp][2], pw[pp][3]);
#pragma unroll
                for (int q = 0; q < 4; ++q) s4[pp] = __dp4a(static_cast<int>(pw[pp][q]), 0x01010101, s4[pp]);
            }
        }
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s4[pp] += __shfl_xor_sync(0xFFFFFFFFu, s4[pp], o);
            if (lane == 0) red_s[warp][pp] = s4[pp];
        }
        __syncthreads();
        if (tid == 0) {
            long long t = 0;
            for (int w = 0; w < kThreads / 32; ++w)
                for (int pp = 0; pp < 4; ++pp) t += static_cast<long long>(red_s[w][pp]) * (1LL << (8 * pp));
            sx_sh = static_cast<double>(t);
        }
        __syncthreads();
        const double sxd = sx_sh, scale = exp2_int(E - 29);
        const int64_t kq = pb.k / 4, nchunk = pb.k / 64;
        const int64_t ntasks = (pb.n + pb.rows - 1) / pb.rows;
        for (;;) {
            int task = 0;
            if (lane == 0) task = atomicAdd(pb.counter, 1);
            task = __shfl_sync(0xFFFFFFFFu, task, 0);
            if (task >= ntasks) break;
            if (pb.rows == 4) row_task_i8<4>(pb, task, kq, nchunk, lane, prm.P4, prm.PQ, sxd, scale, xq);
            else if (pb.rows == 2) row_task_i8<2>(pb, task, kq, nchunk, lane, prm.P4, prm.PQ, sxd, scale, xq);
            else row_task_i8<1>(pb, task, kq, nchunk, lane, prm.P4, prm.PQ, sxd, scale, xq);
        }
        __syncthreads();  // the next matrix overwrites the planes
    }
}

}  // namespace pqv

// ------------------------------------------------------------------- host

static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

constexpr int kMaxBatch = 64;  // matrices per launch (their descriptors travel as parameters)

// Integer mode pre-pass: each distinct activation matrix as signed base-256
// digit planes. Row j of x is scaled by 2^(29 - E), E = floor(log2 max|x_j|),
// and rounded to the nearest integer v (|v| < 2^30; exact for every x within
// 2^22 of the row's largest magnitude, bf16 having 8 significant bits);
// v = d0 + 256 d1 + 65536 d2 + 2^24 d3 with every digit in [-128, 127].
// Plane p of row j is row 4j + p of a [4m][k] int8 matrix, its K order
// inside every group of 16 transposed 4 x 4 like the decoded weights.
// A row is split into `slices` CTAs; each finds the row's max|x| itself
// (the row is small and in L2) and converts its share of 16-element groups.
// fp4 mode: the same fixed point as ten base-9 digit planes of packed e2m1
// nibbles, plane p of row j being row p * mp + j of a [10 mp][k / 2] byte
// matrix (mp = 8 or 16 rows per plane; rows m..mp-1 are zero).
struct XPlanes {
    const uint16_t* x[kMaxBatch];
    int8_t* planes[kMaxBatch];
    int* exps[kMaxBatch];
    int64_t k[kMaxBatch];
    int32_t m, slices;
    int32_t mp;  // fp4 mode: rows per plane (the grid covers mp rows per matrix)
};

template <bool F4>
__global__ void __launch_bounds__(256) xplanes_kernel(const __grid_constant__ XPlanes prm) {
    __shared__ uint32_t red[8];
    __shared__ int e_sh;
    const int rows = F4 ? prm.mp : prm.m;
    const int row = blockIdx.x / prm.slices, slice = blockIdx.x % prm.slices;
    const int xi = row / rows, j = row % rows;
    const int64_t k = prm.k[xi];
    if (F4 && j >= prm.m) {  // padding rows of the planes: zero
        const int64_t rb = k / 2;
        const int64_t words = rb / 16;
        const int64_t w1 = words * (slice + 1) / prm.slices;
        for (int pp = 0; pp < kF4Planes; ++pp) {
            uint4* dst = reinterpret_cast<uint4*>(prm.planes[xi] + (pp * prm.mp + j) * rb);
            for (int64_t i = words * slice / prm.slices + threadIdx.x; i < w1; i += 256)
                dst[i] = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const uint16_t* xr = prm.x[xi] + j * k;
    // max |x| of the row: the bf16 bits with the sign cleared order like the values
    uint32_t mb = 0;
    for (int64_t i = threadIdx.x; i < k / 8; i += 256) {
        const uint4 h = __ldg(reinterpret_cast<const uint4*>(xr) + i);
        const uint32_t a = __vmaxu2(__vmaxu2(h.x & 0x7FFF7FFFu, h.y & 0x7FFF7FFFu),
                                    __vmaxu2(h.z & 0x7FFF7FFFu, h.w & 0x7FFF7FFFu));  // per half
        mb = max(mb, max(a & 0xFFFFu, a >> 16));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mb;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = red[0];
        for (int w = 1; w < 8; ++w) t = max(t, red[w]);
        e_sh = exponent_of_max(t);
        if (slice == 0) prm.exps[xi][j] = e_sh;
    }
    __syncthreads();
    const int E = e_sh;
    const int64_t groups = k / 16;
    const int64_t g1 = groups * (slice + 1) / prm.slices;
    for (int64_t g = groups * slice / prm.slices + threadIdx.x; g < g1; g += 256) {
        const uint4 h0 = reinterpret_cast<const uint4*>(xr + 16 * g)[0];
        const uint4 h1 = reinterpret_cast<const uint4*>(xr + 16 * g)[1];
        const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
        if constexpr (F4) {
            uint32_t w0[kF4Planes], w1[kF4Planes];
            digits16_f4(hw, E, w0, w1);
            const int64_t rb = k / 2;
#pragma unroll
            for (int pp = 0; pp < kF4Planes; ++pp)
                *reinterpret_cast<uint2*>(prm.planes[xi] + (pp * prm.mp + j) * rb + 8 * g) = make_uint2(w0[pp], w1[pp]);
        } else {
            int8_t* pl = prm.planes[xi] + 4 * j * k;
            uint32_t pw[4][4];
            digits16(hw, E, pw);
#pragma unroll
            for (int pp = 0; pp < 4; ++pp)
                *reinterpret_cast<uint4*>(pl + pp * k + 16 * g) = make_uint4(pw[pp][0], pw[pp][1], pw[pp][2], pw[pp][3]);
        }
    }
}

struct Plan {
    int nt;
    int64_t items, blocks;  // over all matrices of the launch
    int grid;
    bool partials;          // some CTA range cuts a row block
};

// Work list of a launch: matrix i's items start at item0[i], its block
// counters at block0[i].
static Plan plan(int64_t m, const pq_gemm_problem_t* pr, int count, int64_t* item0,
                 int64_t* block0, int64_t* nchunks, int mode) {
    Plan pl;
    if (mode == kModeF4) {
        pl.nt = m <= 8 ? 80 : 160;  // ten planes of 8 or 16 rows
    } else {
        const int64_t rows = mode == kModeI8 ? 4 * m : m;  // B rows: activations, or their 4 digit planes
        pl.nt = rows <= 16 ? 16 : rows <= 32 ? 32 : rows <= 64 ? 64 : 128;
    }
    int64_t items = 0, blocks = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t nb = (pr[i].n + kFeat - 1) / kFeat;
        const int64_t nc = (pr[i].k + kChunkK - 1) / kChunkK;
        item0[i] = items;
        block0[i] = blocks;
        nchunks[i] = nc;
        items += nb * nc;
        blocks += nb;
    }
    pl.items = items;
    pl.blocks = blocks;
    const int64_t sms = sm_count();
    pl.grid = static_cast<int>(items < sms ? items : sms);
    pl.partials = false;
    int cur = 0;
    for (int64_t g = 1; g < pl.grid; ++g) {
        const int64_t st = g * items / pl.grid;
        while (cur + 1 < count && st >= item0[cur + 1]) ++cur;
        if ((st - item0[cur]) % nchunks[cur] != 0) pl.partials = true;
    }
    return pl;
}

// y = alpha * (P * D + Q * Sx) for D = sum x (1 + f'/4), Sx = sum x.
static bool coeffs_of(int q, float& P, float& Q) {
    double A, B, factor;
    switch (q) {
        case PQ_SEQ2: A = 2; B = -3; factor = 0.25; break;
        case PQ_SEQ2_B: A = 2; B = -3; factor = 1.0 / 3.0; break;
        case PQ_TERNARY: A = 2; B = -4; factor = 1.0 / 3.0; break;
        case PQ_LSQ2: case PQ_BINARY: A = 1; B = -2; factor = 1.0; break;
        default: return false;
    }
    P = static_cast<float>(4.0 * A * factor);
    Q = static_cast<float>((B - 4.0 * A) * factor);
    return true;
}

// Integer mode: y = alpha * factor * (A * sum x f' + B * Sx) in double.
static bool coeffs_i8(int q, double& P4, double& PQ) {
    double A, B, factor;
    switch (q) {
        case PQ_SEQ2: A = 2; B = -3; factor = 0.25; break;
        case PQ_SEQ2_B: A = 2; B = -3; factor = 1.0 / 3.0; break;
        case PQ_TERNARY: A = 2; B = -4; factor = 1.0 / 3.0; break;
        case PQ_LSQ2: case PQ_BINARY: A = 1; B = -2; factor = 1.0; break;
        default: return false;
    }
    P4 = A * factor;
    PQ = B * factor;
    return true;
}

// Up to 16 activation rows take the exact fixed-point arithmetic (one row
// takes the CUDA-core path when its x fits shared memory): on packed fp4
// MMAs while every k <= 2^20 (the fp32 accumulators then hold exact
// integers), else on 8-bit MMAs (s32 accumulators); more rows take bf16.
static int mode_of(int64_t m, const pq_gemm_problem_t* pr, int count) {
    if (m > 16) return kModeBF16;
    for (int i = 0; i < count; ++i)
        if (pr[i].k > kF4MaxK) return kModeI8;
    return kModeF4;
}

static int64_t round256(int64_t b) { return (b + 255) / 256 * 256; }

// fp4 mode: rows per digit plane.
static int64_t f4_rows(int64_t m) { return m <= 8 ? 8 : 16; }

// Digit planes of one activation matrix: [4m][k] int8 (integer mode) or
// [10 mp][k/2] bytes (fp4 mode); the exponents [m] int32 follow them.
static int64_t planes_bytes(int mode, int64_t m, int64_t k) {
    return mode == kModeF4 ? round256(kF4Planes * f4_rows(m) * (k / 2)) : round256(4 * m * k);
}
static int64_t xplanes_bytes(int mode, int64_t m, int64_t k) {
    return planes_bytes(mode, m, k) + round256(4 * m);
}

static int64_t partial_bytes(const Plan& pl, int64_t m) {
    const int64_t m4 = (m + 3) / 4 * 4;
    return (static_cast<int64_t>(pl.grid) * 2 * kFeat * m4 * 4 + 255) / 256 * 256;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Argument checks of one matrix (no CUDA call).
static pq_status_t check_problem(int64_t m, const pq_gemm_problem_t& pr) {
    if (m < 1 || m > 128 || pr.n < 1 || pr.k < kMinK || pr.k % kMinK) return PQ_ERR_INVALID_ARG;
    if (pr.n > (int64_t{1} << 30) || pr.k > (int64_t{1} << 30)) return PQ_ERR_INVALID_ARG;
    if (!pr.x_bf16 || !pr.packed || !pr.alpha || !pr.y_bf16) return PQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(pr.x_bf16) & 15) ||
        (reinterpret_cast<uintptr_t>(pr.packed) & 15) || (reinterpret_cast<uintptr_t>(pr.y_bf16) & 1))
        return PQ_ERR_MISALIGNED;
    return PQ_OK;
}

// Tensor maps of one matrix: codes [n rows][k/4 bytes] in boxes of 127 rows
// x 128 B, activations [m rows][k] in boxes of nt rows x 64 K, both with the
// 128B swizzle the MMA and the decoders read.
static bool encode_maps(PFN_cuTensorMapEncodeTiled_v12000 enc, int64_t m, int nt, int mode,
                        const pq_gemm_problem_t& pr, Problem& out, const int8_t* planes) {
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(pr.k / 4), static_cast<cuuint64_t>(pr.n)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(pr.k / 4)};
        const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kFeat)};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&out.tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(pr.packed), dims,
                strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    if (planes) {
        // integer mode: digit planes [4m rows][k] int8, boxes of nt rows x 128 K;
        // fp4: [10 mp rows][k/2] bytes, boxes of nt = 10 mp rows x 256 K
        const int64_t row_bytes = mode == kModeF4 ? pr.k / 2 : pr.k;
        const int64_t rows = mode == kModeF4 ? kF4Planes * f4_rows(m) : 4 * m;
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
        const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(nt)};
        const cuuint32_t es[2] = {1, 1};
        return enc(&out.tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(planes), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(pr.k), static_cast<cuuint64_t>(m)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(pr.k * 2)};
        const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(nt)};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&out.tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(pr.x_bf16), dims,
                strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

template <int NT, int MAXP, int MODE>
static cudaError_t launch(const GemmParams<MAXP>& prm, cudaStream_t s) {
    using L = Layout<NT, MODE>;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(
            wq_gemm_kernel<NT, MAXP, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    wq_gemm_kernel<NT, MAXP, MODE><<<prm.c.grid, Roles<MODE>::kThreads, L::kBytes, s>>>(prm);
    pqc::count_launch();
    return cudaGetLastError();
}

// Weights from which one row times a lone matrix takes the integer one-row
// kernel (its x staging costs more per call, its loop less per weight).
constexpr int64_t kIntegerRowWeights = int64_t{1} << 27;

// A single activation row times a lone matrix, x fitting shared memory, takes
// the CUDA-core path (measured faster there; a group of matrices runs faster
// through the integer tensor-core mode, whose pipeline does not restart per
// matrix).
static bool vector_path(int64_t m, const pq_gemm_problem_t* pr, int count) {
    if (m != 1 || count != 1) return false;
    for (int i = 0; i < count; ++i)
        if (pr[i].k > pqv::kMaxK) return false;
    return true;
}

template <int MAXP>
static pq_status_t run_vector(int q, const pq_gemm_problem_t* pr, int count, void* workspace,
                              int64_t ws_bytes, cudaStream_t s) {
    pqv::VecParams<MAXP> V{};
    if (!coeffs_of(q, V.P, V.Q) || !coeffs_i8(q, V.P4, V.PQ)) return PQ_ERR_UNSUPPORTED;
    if (!workspace || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return PQ_ERR_INVALID_ARG;
    int* counters = static_cast<int*>(workspace);
    int64_t maxk = 0;
    for (int i = 0; i < count; ++i) {
        V.prob[i].x = pr[i].x_bf16;
        V.prob[i].codes = pr[i].packed;
        V.prob[i].alpha = pr[i].alpha;
        V.prob[i].y = pr[i].y_bf16;
        V.prob[i].n = pr[i].n;
        V.prob[i].k = pr[i].k;
        V.prob[i].counter = counters + i;
        if (pr[i].k > maxk) maxk = pr[i].k;
    }
    V.count = count;
    const size_t smem = static_cast<size_t>(maxk / 64) * pqv::kChunkF4 * 16;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        const int maxs = static_cast<int>(pqv::kMaxK / 64 * pqv::kChunkF4 * 16);
        if (cudaFuncSetAttribute(pqv::gemv_i8_kernel<MAXP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 maxs) != cudaSuccess ||
            cudaFuncSetAttribute(pqv::gemv_kernel<MAXP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 maxs) != cudaSuccess)
            return PQ_ERR_CUDA;
        attr_set[dev] = true;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pqv::gemv_i8_kernel<MAXP>, pqv::kThreads,
                                                      smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    // rows per task (x loads are shared by the rows of a task): the largest
    // of 4, 2, 1 that still gives about one task per warp of the grid
    const int64_t warps = static_cast<int64_t>(sm_count()) * per_sm * (pqv::kThreads / 32);
    for (int i = 0; i < count; ++i)
        V.prob[i].rows = pr[i].n >= 4 * warps ? 4 : pr[i].n >= 2 * warps ? 2 : 1;
    if (cudaMemsetAsync(counters, 0, static_cast<size_t>(count) * 4, s) != cudaSuccess)
        return PQ_ERR_CUDA;
    // every CTA stages x: no more CTAs than the row tasks keep busy
    int64_t tasks = 0;
    for (int i = 0; i < count; ++i) tasks += (V.prob[i].n + V.prob[i].rows - 1) / V.prob[i].rows;
    const int64_t need_ctas = (tasks + pqv::kThreads / 32 - 1) / (pqv::kThreads / 32);
    const int64_t full = static_cast<int64_t>(sm_count()) * per_sm;
    const int grid = static_cast<int>(need_ctas < full ? need_ctas : full);
    if (pr[0].n * pr[0].k >= kIntegerRowWeights)
        pqv::gemv_i8_kernel<MAXP><<<grid, pqv::kThreads, smem, s>>>(V);
    else
        pqv::gemv_kernel<MAXP><<<grid, pqv::kThreads, smem, s>>>(V);
    pqc::count_launch();
    return cudaGetLastError() == cudaSuccess ? PQ_OK : PQ_ERR_CUDA;
}

static int64_t workspace_bytes(int q, int64_t m, const pq_gemm_problem_t* pr, int count) {
    float P, Q;
    if (!coeffs_of(q, P, Q) || count < 1 || count > kMaxBatch || !pr) return -1;
    for (int i = 0; i < count; ++i) {
        if (m < 1 || m > 128 || pr[i].n < 1 || pr[i].k < kMinK || pr[i].k % kMinK ||
            pr[i].n > (int64_t{1} << 30) || pr[i].k > (int64_t{1} << 30))
            return -1;
    }
    if (vector_path(m, pr, count)) return 256;  // one task counter per matrix
    const int mode = mode_of(m, pr, count);
    int64_t item0[kMaxBatch], block0[kMaxBatch], nchunks[kMaxBatch];
    const Plan pl = plan(m, pr, count, item0, block0, nchunks, mode);
    int64_t b = pl.partials ? partial_bytes(pl, m) + round256(pl.blocks * 4) : 0;
    if (mode != kModeBF16)  // sized as if every matrix had its own activations
        for (int i = 0; i < count; ++i) b += xplanes_bytes(mode, m, pr[i].k);
    return b;
}

template <int MAXP>
static pq_status_t run(int q, int64_t m, const pq_gemm_problem_t* pr, int count, void* workspace,
                       int64_t ws_bytes, cudaStream_t s) {
    GemmParams<MAXP> P{};  // the kernel's parameters (tensor maps included)
    if (!coeffs_of(q, P.c.P, P.c.Q)) return PQ_ERR_UNSUPPORTED;
    if (count < 1 || count > MAXP || !pr) return PQ_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const pq_status_t st = check_problem(m, pr[i]);
        if (st != PQ_OK) return st;
    }
    if (vector_path(m, pr, count)) return run_vector<1>(q, pr, 1, workspace, ws_bytes, s);
    const int mode = mode_of(m, pr, count);
    const bool i8 = mode != kModeBF16;  // fixed-point activations (integer or fp4 MMAs)
    if (i8 && !coeffs_i8(q, P.c.P4, P.c.PQ)) return PQ_ERR_UNSUPPORTED;
    int64_t item0[kMaxBatch], block0[kMaxBatch], nchunks[kMaxBatch];
    const Plan pl = plan(m, pr, count, item0, block0, nchunks, mode);
    const int64_t base = pl.partials ? partial_bytes(pl, m) + round256(pl.blocks * 4) : 0;
    // fixed point: one digit-plane set per distinct activation matrix
    int slot[kMaxBatch];
    int64_t planes_off[kMaxBatch];  // workspace offsets of each set's planes
    int nslots = 0;
    XPlanes X{};
    int64_t need = base;
    if (i8) {
        X.m = static_cast<int32_t>(m);
        X.mp = static_cast<int32_t>(f4_rows(m));
        for (int i = 0; i < count; ++i) {
            int t = 0;
            while (t < nslots && !(X.x[t] == pr[i].x_bf16 && X.k[t] == pr[i].k)) ++t;
            if (t == nslots) {
                X.x[t] = pr[i].x_bf16;
                X.k[t] = pr[i].k;
                planes_off[t] = need;  // exponents follow the planes
                need += xplanes_bytes(mode, m, pr[i].k);
                ++nslots;
            }
            slot[i] = t;
        }
    }
    P.c.m = m;
    P.c.m4 = (m + 3) / 4 * 4;
    P.c.items = pl.items;
    P.c.grid = pl.grid;
    P.c.count = count;
    if (need > 0) {
        if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
            return PQ_ERR_INVALID_ARG;
        P.c.partial = static_cast<float*>(workspace);
        P.c.counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + partial_bytes(pl, m));
        for (int t = 0; t < nslots; ++t) {
            X.planes[t] = static_cast<int8_t*>(workspace) + planes_off[t];
            X.exps[t] = reinterpret_cast<int*>(static_cast<char*>(workspace) + planes_off[t] +
                                               planes_bytes(mode, m, X.k[t]));
        }
    }
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return PQ_ERR_CUDA;
    for (int i = 0; i < count; ++i) {
        Problem& d = P.prob[i];
        if (!encode_maps(enc, m, pl.nt, mode, pr[i], d, i8 ? X.planes[slot[i]] : nullptr)) return PQ_ERR_CUDA;
        d.xexp = i8 ? X.exps[slot[i]] : nullptr;
        d.alpha = pr[i].alpha;
        d.y = pr[i].y_bf16;
        d.n = pr[i].n;
        d.k = pr[i].k;
        d.nchunks = nchunks[i];
        d.item0 = item0[i];
        d.block0 = block0[i];
    }
    if (pl.partials &&
        cudaMemsetAsync(P.c.counters, 0, static_cast<size_t>(pl.blocks) * 4, s) != cudaSuccess)
        return PQ_ERR_CUDA;
    if (i8) {
        // at most one CTA per SM over all rows, each converting >= 64 groups
        int64_t maxk = 0;
        for (int t = 0; t < nslots; ++t) maxk = X.k[t] > maxk ? X.k[t] : maxk;
        const int64_t rows = nslots * (mode == kModeF4 ? X.mp : m);
        int64_t sl = sm_count() / rows;
        const int64_t cap = maxk / (16 * 64);
        sl = sl < cap ? sl : cap;
        X.slices = static_cast<int32_t>(sl < 1 ? 1 : sl);
        if (mode == kModeF4)
            xplanes_kernel<true><<<static_cast<int>(rows * X.slices), 256, 0, s>>>(X);
        else
            xplanes_kernel<false><<<static_cast<int>(rows * X.slices), 256, 0, s>>>(X);
        pqc::count_launch();
        if (cudaGetLastError() != cudaSuccess) return PQ_ERR_CUDA;
    }
    cudaError_t e;
    switch (pl.nt * 4 + mode) {
        case 80 * 4 + kModeF4: e = launch<80, MAXP, kModeF4>(P, s); break;
        case 160 * 4 + kModeF4: e = launch<160, MAXP, kModeF4>(P, s); break;
        case 16 * 4 + kModeI8: e = launch<16, MAXP, kModeI8>(P, s); break;
        case 32 * 4 + kModeI8: e = launch<32, MAXP, kModeI8>(P, s); break;
        case 64 * 4 + kModeI8: e = launch<64, MAXP, kModeI8>(P, s); break;
        case 16 * 4 + kModeBF16: e = launch<16, MAXP, kModeBF16>(P, s); break;
        case 32 * 4 + kModeBF16: e = launch<32, MAXP, kModeBF16>(P, s); break;
        case 64 * 4 + kModeBF16: e = launch<64, MAXP, kModeBF16>(P, s); break;
        default: e = launch<128, MAXP, kModeBF16>(P, s); break;
    }
    return e == cudaSuccess ? PQ_OK : PQ_ERR_CUDA;
}

}  // namespace pqg

using namespace pqg;

extern "C" {

int64_t pq_wq_gemm_workspace_bytes(pq_quant_t q, int64_t m, int64_t n, int64_t k) {
    pq_gemm_problem_t pr = {};
    pr.n = n;
    pr.k = k;
    return workspace_bytes(q, m, &pr, 1);
}

int64_t pq_wq_gemm_batch_workspace_bytes(pq_quant_t q, int64_t m, int32_t count,
                                         const pq_gemm_problem_t* problems) {
    return workspace_bytes(q, m, problems, count);
}

pq_status_t pq_wq_gemm(pq_quant_t q, int64_t m, int64_t n, int64_t k, const uint16_t* x_bf16,
                       const uint8_t* packed, const float* alpha, uint16_t* y_bf16, void* workspace,
                       int64_t workspace_bytes, void* stream) {
    pq_gemm_problem_t pr;
    pr.n = n;
    pr.k = k;
    pr.x_bf16 = x_bf16;
    pr.packed = packed;
    pr.alpha = alpha;
    pr.y_bf16 = y_bf16;
    return run<1>(q, m, &pr, 1, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

pq_status_t pq_wq_gemm_batch(pq_quant_t q, int64_t m, int32_t count,
                             const pq_gemm_problem_t* problems, void* workspace,
                             int64_t workspace_bytes, void* stream) {
    return run<kMaxBatch>(q, m, problems, count, workspace, workspace_bytes,
                          static_cast<cudaStream_t>(stream));
}

int pq_device_status(void) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return PQ_ERR_CUDA;
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
        return PQ_ERR_TIMEOUT;
    }
    return PQ_OK;
}

pq_status_t pq_debug_abort_waits(int on) {
    const int v = on ? 1 : 0;
    return cudaMemcpyToSymbol(g_force_abort, &v, sizeof(v)) == cudaSuccess ? PQ_OK : PQ_ERR_CUDA;
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
    float P, Q;
    if (!coeffs_of(q, P, Q)) return PQ_ERR_UNSUPPORTED;
    if (m < 1 || m > 128 || n < 1 || k < kMinK || k % kMinK || !x_bf16 || !packed || !alpha ||
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
