// Test helper, not part of the library: x = w / alpha_row by CUDA's IEEE
// round-to-nearest division intrinsic (__fdiv_rn), as the reference for the
// library's own division routine in the dense division test. It also draws
// the random operands on the device from a counter-based hash, so that a
// billion pairs cost no host work.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__global__ void fdiv_ref_kernel(const float* __restrict__ w, const float* __restrict__ alpha,
                                float* __restrict__ x, int64_t rows, int64_t cols) {
    const int64_t n = rows * cols;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        x[i] = __fdiv_rn(w[i], alpha[i / cols]);
}

// splitmix64 finaliser of (seed, index): one 64-bit draw per index.
__device__ __forceinline__ uint64_t mix(uint64_t seed, uint64_t i) {
    uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Bit patterns of finite fp32 values. mode 0: any finite value (every
// exponent, subnormals and zeros included); mode 1: |value| in [2^-60, 2^61)
// (biased exponents 67..187). positive != 0 makes the value positive and
// nonzero (a scale).
__global__ void draw_kernel(uint32_t* __restrict__ out, int64_t n, uint64_t seed, int mode,
                            int positive) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint64_t r = mix(seed, static_cast<uint64_t>(i));
        uint32_t sign = static_cast<uint32_t>(r >> 63) << 31;
        uint32_t mant = static_cast<uint32_t>(r) & 0x7FFFFFu;
        uint32_t e = static_cast<uint32_t>(r >> 32) & 0xFFu;
        if (mode == 0) {
            if (e == 0xFFu) e = static_cast<uint32_t>(r >> 40) % 255u;  // finite
        } else {
            e = 67u + static_cast<uint32_t>((r >> 32) % 121u);
        }
        if (positive) {
            sign = 0;
            if (e == 0 && mant == 0) mant = 1;  // smallest subnormal, not zero
        }
        out[i] = sign | (e << 23) | mant;
    }
}

}  // namespace

extern "C" int fdiv_ref(const float* w, const float* alpha, float* x, int64_t rows,
                        int64_t cols, void* stream) {
    if (rows <= 0 || cols <= 0) return 0;
    fdiv_ref_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(w, alpha, x, rows, cols);
    return static_cast<int>(cudaGetLastError());
}

extern "C" int fdiv_draw(uint32_t* out, int64_t n, uint64_t seed, int mode, int positive,
                         void* stream) {
    if (n <= 0) return 0;
    draw_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(out, n, seed, mode, positive);
    return static_cast<int>(cudaGetLastError());
}
