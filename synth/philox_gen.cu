// philox_gen.cu -- seeded synthetic inputs on the GPU (gradients, master
// weights, non-finite injections).  Part of the input generator only: it
// holds none of the optimizer step's arithmetic, and the step's library does
// not link it.  The numpy twin in synth/__init__.py draws the same Philox
// integers (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3", SC'11).
//
// Counter = (block_lo, block_hi, step, 0), key = (seed, stream); see the
// Python module docstring for the stream layout.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; r++) {
        if (r) { k0 += W0; k1 += W1; }
        const uint32_t hi0 = __umulhi(M0, c[0]), lo0 = M0 * c[0];
        const uint32_t hi1 = __umulhi(M1, c[2]), lo1 = M1 * c[2];
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    }
}

__device__ __forceinline__ double uni(uint32_t x) { return ((double)(x >> 8) + 0.5) * (1.0 / 16777216.0); }

__device__ __forceinline__ void box_muller(uint32_t a, uint32_t b, double& z0, double& z1) {
    const double r = sqrt(-2.0 * log(uni(a)));
    double s, c;
    sincospi(2.0 * uni(b), &s, &c);
    z0 = r * c;
    z1 = r * s;
}

__device__ __forceinline__ uint16_t to16(float x, int bf16) {
    return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(x)) : __half_as_ushort(__float2half_rn(x));
}

__global__ void normal16_kernel(uint16_t* out, unsigned long long n, unsigned long long start, float sigma,
                                float scale, uint32_t seed, uint32_t stream, uint32_t step, int bf16) {
    const unsigned long long nb = (start + n + 3) / 4;
    for (unsigned long long b = start / 4 + blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; b < nb;
         b += (unsigned long long)gridDim.x * blockDim.x) {
        uint32_t c[4] = {(uint32_t)b, (uint32_t)(b >> 32), step, 0u};
        philox4x32_10(c, seed, stream);
        double z[4];
        box_muller(c[0], c[1], z[0], z[1]);
        box_muller(c[2], c[3], z[2], z[3]);
#pragma unroll
        for (int l = 0; l < 4; l++) {
            const unsigned long long i = b * 4 + l;
            if (i < start || i >= start + n) continue;
            const float v = ((float)z[l] * sigma) * scale;
            out[i - start] = to16(v, bf16);
        }
    }
}

__global__ void normal32_kernel(float* out, unsigned long long n, unsigned long long start, float sigma,
                                uint32_t seed, uint32_t stream, uint32_t step) {
    const unsigned long long nb = (start + n + 3) / 4;
    for (unsigned long long b = start / 4 + blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; b < nb;
         b += (unsigned long long)gridDim.x * blockDim.x) {
        uint32_t c[4] = {(uint32_t)b, (uint32_t)(b >> 32), step, 0u};
        philox4x32_10(c, seed, stream);
        double z[4];
        box_muller(c[0], c[1], z[0], z[1]);
        box_muller(c[2], c[3], z[2], z[3]);
#pragma unroll
        for (int l = 0; l < 4; l++) {
            const unsigned long long i = b * 4 + l;
            if (i < start || i >= start + n) continue;
            out[i - start] = (float)z[l] * sigma;
        }
    }
}

__global__ void t3_16_kernel(uint16_t* out, unsigned long long n, unsigned long long start, float scale,
                             uint32_t seed, uint32_t stream, uint32_t step, int bf16) {
    for (unsigned long long j = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; j < n;
         j += (unsigned long long)gridDim.x * blockDim.x) {
        const unsigned long long i = start + j;
        uint32_t c[4] = {(uint32_t)i, (uint32_t)(i >> 32), step, 0u};
        philox4x32_10(c, seed, stream);
        double z0, z1, z2, z3;
        box_muller(c[0], c[1], z0, z1);
        box_muller(c[2], c[3], z2, z3);
        const double t = z0 / sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0);
        out[j] = to16((float)t * scale, bf16);
    }
}

__global__ void rate_inject_kernel(uint16_t* out, unsigned long long n, unsigned long long start, uint32_t thresh,
                                   uint32_t seed, uint32_t stream, uint32_t step, int bf16,
                                   unsigned long long* hits) {
    const uint16_t codes16[3] = {0x7c00u, 0x7e00u, 0xfc00u};
    const uint16_t codesbf[3] = {0x7f80u, 0x7fc0u, 0xff80u};
    unsigned long long mine = 0;
    for (unsigned long long j = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; j < n;
         j += (unsigned long long)gridDim.x * blockDim.x) {
        const unsigned long long i = start + j;
        uint32_t c[4] = {(uint32_t)i, (uint32_t)(i >> 32), step, 0u};
        philox4x32_10(c, seed, stream);
        if (c[0] < thresh) {
            const uint32_t kind = c[1] % 3u;
            out[j] = bf16 ? codesbf[kind] : codes16[kind];
            mine++;
        }
    }
    if (mine) atomicAdd(hits, mine);
}

__global__ void raw_kernel(uint32_t* out, unsigned long long nblocks, uint32_t step, uint32_t seed, uint32_t stream) {
    for (unsigned long long b = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; b < nblocks;
         b += (unsigned long long)gridDim.x * blockDim.x) {
        uint32_t c[4] = {(uint32_t)b, (uint32_t)(b >> 32), step, 0u};
        philox4x32_10(c, seed, stream);
        for (int l = 0; l < 4; l++) out[4 * b + l] = c[l];
    }
}

int grid_of(unsigned long long work) {
    unsigned long long g = (work + 255) / 256;
    const unsigned long long cap = 148ull * 16;
    if (g > cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

extern "C" {

int synth_normal16(void* out, unsigned long long n, unsigned long long start, float sigma, float scale,
                   uint32_t seed, uint32_t stream, uint32_t step, int bf16, void* st) {
    if (n == 0) return 0;
    normal16_kernel<<<grid_of(n / 4 + 1), 256, 0, (cudaStream_t)st>>>((uint16_t*)out, n, start, sigma, scale, seed,
                                                                      stream, step, bf16);
    return (int)cudaGetLastError();
}

int synth_normal32(void* out, unsigned long long n, unsigned long long start, float sigma, uint32_t seed,
                   uint32_t stream, uint32_t step, void* st) {
    if (n == 0) return 0;
    normal32_kernel<<<grid_of(n / 4 + 1), 256, 0, (cudaStream_t)st>>>((float*)out, n, start, sigma, seed, stream,
                                                                      step);
    return (int)cudaGetLastError();
}

int synth_t3_16(void* out, unsigned long long n, unsigned long long start, float scale, uint32_t seed,
                uint32_t stream, uint32_t step, int bf16, void* st) {
    if (n == 0) return 0;
    t3_16_kernel<<<grid_of(n), 256, 0, (cudaStream_t)st>>>((uint16_t*)out, n, start, scale, seed, stream, step, bf16);
    return (int)cudaGetLastError();
}

int synth_rate_inject16(void* out, unsigned long long n, unsigned long long start, uint32_t thresh, uint32_t seed,
                        uint32_t stream, uint32_t step, int bf16, void* hits_dev, void* st) {
    if (n == 0) return 0;
    rate_inject_kernel<<<grid_of(n), 256, 0, (cudaStream_t)st>>>((uint16_t*)out, n, start, thresh, seed, stream,
                                                                  step, bf16, (unsigned long long*)hits_dev);
    return (int)cudaGetLastError();
}

int synth_philox_raw(void* out, unsigned long long nblocks, uint32_t step, uint32_t seed, uint32_t stream, void* st) {
    if (nblocks == 0) return 0;
    raw_kernel<<<grid_of(nblocks), 256, 0, (cudaStream_t)st>>>((uint32_t*)out, nblocks, step, seed, stream);
    return (int)cudaGetLastError();
}

}  // extern "C"
