// neox_common.cuh -- device arithmetic and host helpers shared by the flat-shard
// step (neox_shard.cu) and the multi-tensor step (neox_multi.cu) of
// libneoxshard.so.  Everything here is inline / internal to each translation
// unit; both units therefore run the same per-element arithmetic.
#pragma once

#include "neox_shard.h"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <unordered_map>

namespace {

constexpr int kMaxGrads = 64;
constexpr int kThreads1 = 512;   // pass-1 block
constexpr int kUnroll1 = 4;      // pass-1 vectors in flight per thread
constexpr int kThreads3 = 256;   // pass-2 block
constexpr int kChunk3 = 2;       // pass-2 (AdamW) vectors per thread in each chunk taken from the counter
constexpr int kUnrollSgd = 4;    // pass-2 vectors in flight per thread (SGD): measured 6.25 TB/s against 5.83 at 1
constexpr int kMaxBlocksPerSm = 32;

struct GradPtrs {
    const uint16_t* p[kMaxGrads];
    __device__ __forceinline__ const uint16_t* operator[](int k) const { return p[k]; }
};

// The K gradient pointers of one tensor in a device-resident table.
struct GradTab {
    const uint16_t* const* t;
    int base;
    __device__ __forceinline__ const uint16_t* operator[](int k) const { return t[base + k]; }
};

// Device-resident scalars of one shard (64 bytes).  `scale`, `good`, `t` are
// the scaler / step state; the rest describe the most recent step.
struct __align__(64) DevScalars {
    double sumsq;          // sum of squared unscaled grads of the last step
    float scale;           // S the next step's grads carry
    int32_t good;          // consecutive applied steps
    long long t;           // applied steps
    int32_t overflow;      // last step overflowed
    float coef;            // clip coefficient of the last step
    float scale_used;      // S the last step's grads carried
    float norm;            // pre-clip norm of the last step (+inf on overflow)
    unsigned int blocks_done;  // pass-1 ticket counter, back to 0 after each step
    float step_size;       // device-computed fl32(lr / bc1) of the last step (asynchronous steps)
    float bc2_sqrt;        // device-computed fl32(sqrt(bc2)) of the last step (asynchronous steps)
    float lr;              // learning rate of the last step (asynchronous steps)
    int32_t hyst;          // overflows still tolerated before the next back-off
    unsigned int chunk_next;   // pass-2 work counter: zeroed before every pass 2
};
static_assert(sizeof(DevScalars) == 64, "DevScalars is one 64-byte block");

// Which elements use vectors: [0, head) scalar, [head, head + nvec*VEC)
// vectors of VEC, [tail0, n) scalar.
struct Layout {
    unsigned long long n, head, nvec, tail0;
};

struct ScalerArgs {
    double post;          // K / predivide
    float inv_pre;        // fl32(1 / predivide)
    float clip;           // <= 0: off
    float factor, min_scale;
    int32_t window;
    int32_t hyst_full;    // max(hysteresis, 1): the count after a growth
    // asynchronous steps: the bias corrections are formed on the device from
    // the device step count, and the result is written to `result`
    int32_t device_bc;
    float lr, beta1, beta2;
    const float* lr_ptr;       // when non-NULL, the learning rate is read here
    neox_step_result* result;  // device-accessible; NULL = not written
    // split step: pass 1 writes {sum of squares, non-finite flag} here and
    // takes no decision (the ranks' statistics are all-reduced first)
    double* stats_out;
};

// Extra destinations of the 16-bit working weights (e.g. this rank's slice
// of the full weight buffer on every peer), written with the same bytes as
// the shard's own copy.
constexpr int kMaxWeightCopies = 8;
struct WeightCopies {
    uint16_t* p[kMaxWeightCopies];
    int n;
};

struct AdamArgs {
    float lr, b1, b2, omb1, omb2, eps;
    float step_size;      // fl32(lr / bc1) for t+1
    float bcs;            // fl32(sqrt(bc2)) for t+1
    float inv_pre;
    int32_t device_bc;    // take lr, step_size and bcs from the device scalars
    double post;
};

// ---------------------------------------------------------------- 16-bit types
struct F16 {
    static __device__ __forceinline__ float dec(uint16_t h) { return __half2float(__ushort_as_half(h)); }
    static __device__ __forceinline__ uint16_t enc(float f) { return __half_as_ushort(__float2half_rn(f)); }
    static __device__ __forceinline__ uint32_t enc2(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};
struct BF16 {
    static __device__ __forceinline__ float dec(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }
    static __device__ __forceinline__ uint16_t enc(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
    static __device__ __forceinline__ uint32_t enc2(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

// ---------------------------------------------------------------- vector I/O
// VEC 16-bit values starting at p (aligned to 2*VEC bytes), read-only data.
template <int VEC>
__device__ __forceinline__ void ld16(const uint16_t* p, uint16_t (&o)[VEC]) {
    if constexpr (VEC == 8) {
        uint4 r = __ldcs(reinterpret_cast<const uint4*>(p));
        uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; i++) { o[2 * i] = uint16_t(w[i]); o[2 * i + 1] = uint16_t(w[i] >> 16); }
    } else if constexpr (VEC == 4) {
        uint2 r = __ldcs(reinterpret_cast<const uint2*>(p));
        o[0] = uint16_t(r.x); o[1] = uint16_t(r.x >> 16); o[2] = uint16_t(r.y); o[3] = uint16_t(r.y >> 16);
    } else if constexpr (VEC == 2) {
        uint32_t r = __ldcs(reinterpret_cast<const unsigned int*>(p));
        o[0] = uint16_t(r); o[1] = uint16_t(r >> 16);
    } else {
        o[0] = __ldcs(reinterpret_cast<const unsigned short*>(p));
    }
}

template <class W, int VEC>
__device__ __forceinline__ void st16(uint16_t* p, const float (&x)[VEC]) {
    if constexpr (VEC == 8) {
        uint4 r = make_uint4(W::enc2(x[0], x[1]), W::enc2(x[2], x[3]), W::enc2(x[4], x[5]), W::enc2(x[6], x[7]));
        __stcs(reinterpret_cast<uint4*>(p), r);
    } else if constexpr (VEC == 4) {
        uint2 r = make_uint2(W::enc2(x[0], x[1]), W::enc2(x[2], x[3]));
        __stcs(reinterpret_cast<uint2*>(p), r);
    } else if constexpr (VEC == 2) {
        __stcs(reinterpret_cast<unsigned int*>(p), W::enc2(x[0], x[1]));
    } else {
        __stcs(reinterpret_cast<unsigned short*>(p), W::enc(x[0]));
    }
}

// VEC FP32 values at p (16-byte aligned when VEC >= 4).
template <int VEC>
__device__ __forceinline__ void ld32(const float* p, float (&o)[VEC]) {
    if constexpr (VEC >= 4) {
#pragma unroll
        for (int q = 0; q < VEC / 4; q++) {
            float4 r = __ldcs(reinterpret_cast<const float4*>(p) + q);
            o[4 * q] = r.x; o[4 * q + 1] = r.y; o[4 * q + 2] = r.z; o[4 * q + 3] = r.w;
        }
    } else if constexpr (VEC == 2) {
        float2 r = __ldcs(reinterpret_cast<const float2*>(p));
        o[0] = r.x; o[1] = r.y;
    } else {
        o[0] = __ldcs(p);
    }
}

template <int VEC>
__device__ __forceinline__ void st32(float* p, const float (&x)[VEC]) {
    if constexpr (VEC >= 4) {
#pragma unroll
        for (int q = 0; q < VEC / 4; q++)
            __stcs(reinterpret_cast<float4*>(p) + q, make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]));
    } else if constexpr (VEC == 2) {
        __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
    } else {
        __stcs(p, x[0]);
    }
}

__device__ __forceinline__ bool not_finite(float x) {
    return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

// Unscaled gradients of VEC consecutive elements from global index i:
// a = sum_k fl32(g_k * inv_pre) in buffer order (starting from +0, as a
// sequential sum does), then fl32(a * inv_us).
template <class G, int VEC, class PT>
__device__ __forceinline__ void ingest(const PT& gp, int K, unsigned long long i,
                                       float inv_pre, float inv_us, float (&g)[VEC]) {
#pragma unroll
    for (int e = 0; e < VEC; e++) g[e] = 0.0f;
    const bool pre1 = inv_pre == 1.0f;  // x * 1 == x exactly: skip the multiply
    for (int k = 0; k < K; k++) {
        uint16_t h[VEC];
        ld16<VEC>(gp[k] + i, h);
        if (pre1) {
#pragma unroll
            for (int e = 0; e < VEC; e++) g[e] = __fadd_rn(g[e], G::dec(h[e]));
        } else {
#pragma unroll
            for (int e = 0; e < VEC; e++) g[e] = __fadd_rn(g[e], __fmul_rn(G::dec(h[e]), inv_pre));
        }
    }
#pragma unroll
    for (int e = 0; e < VEC; e++) g[e] = __fmul_rn(g[e], inv_us);
}

// U vectors at global indices i0, i0 + di, ..., ingested together: for every
// buffer the U loads are issued before any of them is used, so each thread
// keeps U 16-byte requests in flight.  Per element the arithmetic (and its
// order over buffers) is that of ingest().
template <class G, int VEC, int U, class PT>
__device__ __forceinline__ void ingest_batch(const PT& gp, int K, unsigned long long i0, unsigned long long di,
                                             float inv_pre, float inv_us, float (&g)[U][VEC]) {
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < VEC; e++) g[u][e] = 0.0f;
    const bool pre1 = inv_pre == 1.0f;  // x * 1 == x exactly: skip the multiply
    for (int k = 0; k < K; k++) {
        uint16_t h[U][VEC];
#pragma unroll
        for (int u = 0; u < U; u++) ld16<VEC>(gp[k] + i0 + u * di, h[u]);
        if (pre1) {
#pragma unroll
            for (int u = 0; u < U; u++)
#pragma unroll
                for (int e = 0; e < VEC; e++) g[u][e] = __fadd_rn(g[u][e], G::dec(h[u][e]));
        } else {
#pragma unroll
            for (int u = 0; u < U; u++)
#pragma unroll
                for (int e = 0; e < VEC; e++) g[u][e] = __fadd_rn(g[u][e], __fmul_rn(G::dec(h[u][e]), inv_pre));
        }
    }
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < VEC; e++) g[u][e] = __fmul_rn(g[u][e], inv_us);
}

// ingest_batch with the buffers taken two at a time: the 2U loads of buffers
// k and k + 1 are issued before either is used (for K > 1 and a short U this
// doubles the bytes each thread keeps in flight).  Per element the sum still
// runs over the buffers in order, so the result is ingest_batch's.
template <class G, int VEC, int U, class PT>
__device__ __forceinline__ void ingest_batch_pairs(const PT& gp, int K, unsigned long long i0, unsigned long long di,
                                                   float inv_pre, float inv_us, float (&g)[U][VEC]) {
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < VEC; e++) g[u][e] = 0.0f;
    const bool pre1 = inv_pre == 1.0f;
    int k = 0;
    for (; k + 1 < K; k += 2) {
        uint16_t h0[U][VEC], h1[U][VEC];
#pragma unroll
        for (int u = 0; u < U; u++) ld16<VEC>(gp[k] + i0 + u * di, h0[u]);
#pragma unroll
        for (int u = 0; u < U; u++) ld16<VEC>(gp[k + 1] + i0 + u * di, h1[u]);
#pragma unroll
        for (int u = 0; u < U; u++)
#pragma unroll
            for (int e = 0; e < VEC; e++) {
                g[u][e] = __fadd_rn(g[u][e], pre1 ? G::dec(h0[u][e]) : __fmul_rn(G::dec(h0[u][e]), inv_pre));
                g[u][e] = __fadd_rn(g[u][e], pre1 ? G::dec(h1[u][e]) : __fmul_rn(G::dec(h1[u][e]), inv_pre));
            }
    }
    if (k < K) {
        uint16_t h[U][VEC];
#pragma unroll
        for (int u = 0; u < U; u++) ld16<VEC>(gp[k] + i0 + u * di, h[u]);
#pragma unroll
        for (int u = 0; u < U; u++)
#pragma unroll
            for (int e = 0; e < VEC; e++)
                g[u][e] = __fadd_rn(g[u][e], pre1 ? G::dec(h[u][e]) : __fmul_rn(G::dec(h[u][e]), inv_pre));
    }
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < VEC; e++) g[u][e] = __fmul_rn(g[u][e], inv_us);
}

// U split vectors: vector u is the 4 elements at i0 + u*di and the 4 at
// i0 + u*di + 128 (g[u][0..3] and g[u][4..7]).  All 2U loads of a buffer are
// issued before any is used.  Per element the arithmetic is ingest()'s, over
// the buffers in order.
template <class G, int U, class PT>
__device__ __forceinline__ void ingest_halves(const PT& gp, int K, unsigned long long i0, unsigned long long di,
                                              float inv_pre, float inv_us, float (&g)[U][8]) {
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < 8; e++) g[u][e] = 0.0f;
    const bool pre1 = inv_pre == 1.0f;
    for (int k = 0; k < K; k++) {
        uint16_t a[U][4], b[U][4];
#pragma unroll
        for (int u = 0; u < U; u++) {
            ld16<4>(gp[k] + i0 + u * di, a[u]);
            ld16<4>(gp[k] + i0 + u * di + 128, b[u]);
        }
#pragma unroll
        for (int u = 0; u < U; u++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                g[u][e] = __fadd_rn(g[u][e], pre1 ? G::dec(a[u][e]) : __fmul_rn(G::dec(a[u][e]), inv_pre));
                g[u][4 + e] = __fadd_rn(g[u][4 + e], pre1 ? G::dec(b[u][e]) : __fmul_rn(G::dec(b[u][e]), inv_pre));
            }
    }
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < 8; e++) g[u][e] = __fmul_rn(g[u][e], inv_us);
}

// ingest_batch for the last strides of a range: vector u is ingested only
// when ok[u]; the loads of all valid vectors are still issued together.
template <class G, int VEC, int U, class PT>
__device__ __forceinline__ void ingest_batch_pred(const PT& gp, int K, unsigned long long i0, unsigned long long di,
                                                  const bool (&ok)[U], float inv_pre, float inv_us,
                                                  float (&g)[U][VEC]) {
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < VEC; e++) g[u][e] = 0.0f;
    const bool pre1 = inv_pre == 1.0f;
    for (int k = 0; k < K; k++) {
        uint16_t h[U][VEC];
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (ok[u]) ld16<VEC>(gp[k] + i0 + u * di, h[u]);
            else {
#pragma unroll
                for (int e = 0; e < VEC; e++) h[u][e] = 0;
            }
        }
#pragma unroll
        for (int u = 0; u < U; u++)
#pragma unroll
            for (int e = 0; e < VEC; e++)
                g[u][e] = __fadd_rn(g[u][e], pre1 ? G::dec(h[u][e]) : __fmul_rn(G::dec(h[u][e]), inv_pre));
    }
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < VEC; e++) g[u][e] = __fmul_rn(g[u][e], inv_us);
}

__device__ __forceinline__ float unscale_factor(double post, float scale) {
    return (float)(1.0 / (post * (double)scale));
}

// Sum of squares of a vector (FP32 within the vector) and the non-finite
// flag.  A sum of squares is finite exactly when every element is finite and
// no square or partial sum passes FP32's range, so one test per vector
// replaces a test per element; only a vector that fails it looks at its
// elements (and, when they are all finite, redoes the sum in FP64).
template <int VEC>
__device__ __forceinline__ double vec_sumsq(const float (&g)[VEC], int& bad) {
    float q = 0.0f;
#pragma unroll
    for (int e = 0; e < VEC; e++) q = __fmaf_rn(g[e], g[e], q);
    if (!(q <= 3.40282346638528859812e+38f)) {
        int vb = 0;
#pragma unroll
        for (int e = 0; e < VEC; e++) vb |= not_finite(g[e]);
        bad |= vb;
        if (!vb) {
            double d = 0.0;
#pragma unroll
            for (int e = 0; e < VEC; e++) d += (double)g[e] * (double)g[e];
            return d;
        }
    }
    return (double)q;
}

// Block-wide reduction of (double, int-or) with a fixed shape.
template <int THREADS>
__device__ __forceinline__ void block_reduce(double& s, int& bad, double* sh_s, int* sh_b) {
    const unsigned full = 0xffffffffu;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        s += __shfl_down_sync(full, s, off);
        bad |= __shfl_down_sync(full, bad, off);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { sh_s[warp] = s; sh_b[warp] = bad; }
    __syncthreads();
    if (warp == 0) {
        constexpr int NW = THREADS / 32;
        s = lane < NW ? sh_s[lane] : 0.0;
        bad = lane < NW ? sh_b[lane] : 0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            s += __shfl_down_sync(full, s, off);
            bad |= __shfl_down_sync(full, bad, off);
        }
    }
}

// ---------------------------------------------------------------- pass 1
// The end of pass 1, shared by every pass-1 kernel: the block's partial sum
// and flag, a ticket, and -- in the last block to finish -- the fixed-order
// reduction of all partials and the step's scalar decisions (overflow, norm,
// loss scaler, clip coefficient, applied-step count; for asynchronous steps
// also the bias corrections and the caller's result record).  No spinning:
// every block but the last simply returns.
// The scalar decisions of a step from its global sum of squares `s` and
// non-finite flag `bad`: overflow, norm, dynamic loss scaler, clip
// coefficient, applied-step count; for asynchronous steps also the bias
// corrections and the caller's result record.  One thread.
__device__ __forceinline__ void decide_step(DevScalars* __restrict__ sc, const ScalerArgs& sa, double s, int bad) {
    int overflow = bad != 0;
    const double norm = sqrt(s);
    if (!overflow && !isfinite(norm)) overflow = 1;
    float S = sc->scale;
    int good = sc->good;
    long long t = sc->t;
    sc->scale_used = S;
    sc->sumsq = s;
    sc->overflow = overflow;
    if (overflow) {
        int h = sc->hyst;
        if (h > 0) h -= 1;
        sc->hyst = h;
        if (h == 0) {
            const float d = S / sa.factor;
            S = d > sa.min_scale ? d : sa.min_scale;
        }
        good = 0;
        sc->coef = 0.0f;
        sc->norm = __int_as_float(0x7f800000);
    } else {
        good += 1;
        if (good >= sa.window) {
            const float u = S * sa.factor;
            if (!not_finite(u)) S = u;
            good = 0;
            sc->hyst = sa.hyst_full;
        }
        t += 1;
        float c = 1.0f;
        if (sa.clip > 0.0f) {
            const double cd = (double)sa.clip / (norm + 1e-6);
            if (cd < 1.0) c = (float)cd;
        }
        sc->coef = c;
        sc->norm = (float)norm;
    }
    sc->scale = S;
    sc->good = good;
    sc->t = t;
    if (sa.device_bc) {
        const float lr = sa.lr_ptr ? *sa.lr_ptr : sa.lr;
        sc->lr = lr;
        if (!overflow) {
            const double bc1 = 1.0 - pow((double)sa.beta1, (double)t);
            const double bc2 = 1.0 - pow((double)sa.beta2, (double)t);
            sc->step_size = (float)((double)lr / bc1);
            sc->bc2_sqrt = (float)sqrt(bc2);
        }
        if (sa.result) {
            neox_step_result* r = sa.result;
            r->overflow = overflow;
            r->grad_norm = sc->norm;
            r->clip_coef = sc->coef;
            r->loss_scale = sc->scale_used;
            r->loss_scale_next = S;
            r->good_steps = good;
            r->applied_steps = t;
        }
    }
}

template <int THREADS>
__device__ __forceinline__ void finish_pass1(double s, int bad, double* __restrict__ part_s, int* __restrict__ part_b,
                                             DevScalars* __restrict__ sc, const ScalerArgs& sa, double* sh_s, int* sh_b,
                                             bool* is_last_sh) {
    bool& is_last = *is_last_sh;
    // Let the update kernel's blocks start their prologue as this grid winds
    // down; they wait (griddepcontrol.wait) for this grid's completion before
    // reading anything it writes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    block_reduce<THREADS>(s, bad, sh_s, sh_b);
    if (threadIdx.x == 0) {
        part_s[blockIdx.x] = s;
        part_b[blockIdx.x] = bad;
        __threadfence();
        const unsigned ticket = atomicAdd(&sc->blocks_done, 1u);
        is_last = (ticket == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;

    // Last block: every other block's partial is visible (each fenced before
    // taking its ticket).  Reduce them in a fixed order.
    __threadfence();
    s = 0.0;
    bad = 0;
    for (unsigned j = threadIdx.x; j < gridDim.x; j += THREADS) {
        s += __ldcg(part_s + j);
        bad |= __ldcg(part_b + j);
    }
    __syncthreads();
    block_reduce<THREADS>(s, bad, sh_s, sh_b);
    if (threadIdx.x != 0) return;

    if (sa.stats_out) {  // split step: publish the statistics, decide later
        sa.stats_out[0] = s;
        sa.stats_out[1] = bad ? 1.0 : 0.0;
    } else {
        decide_step(sc, sa, s, bad);
    }
    sc->blocks_done = 0;
    sc->chunk_next = 0;  // for the pass 2 that follows (it waits for this grid to finish)
}

template <int VEC>
__device__ __forceinline__ void adam_vec(const float (&g)[VEC], const float (&keep)[VEC], float c,
                                         const AdamArgs& a, float (&p)[VEC], float (&m)[VEC], float (&v)[VEC]) {
#pragma unroll
    for (int e = 0; e < VEC; e++) {
        const float gh = __fmul_rn(g[e], c);
        const float mj = __fadd_rn(__fmul_rn(a.b1, m[e]), __fmul_rn(a.omb1, gh));
        const float gg = __fmul_rn(a.omb2, gh);
        const float vj = __fadd_rn(__fmul_rn(a.b2, v[e]), __fmul_rn(gg, gh));
        const float den = __fadd_rn(__fdiv_rn(__fsqrt_rn(vj), a.bcs), a.eps);
        float pj = __fmul_rn(p[e], keep[e]);
        const float upd = __fdiv_rn(mj, den);
        pj = __fsub_rn(pj, __fmul_rn(a.step_size, upd));
        m[e] = mj;
        v[e] = vj;
        p[e] = pj;
    }
}

// Plain SGD (no momentum) with the decoupled decay: p*keep - lr*(g*c).
template <int VEC>
__device__ __forceinline__ void sgd_vec(const float (&g)[VEC], const float (&keep)[VEC], float c, float lr,
                                        float (&p)[VEC]) {
#pragma unroll
    for (int e = 0; e < VEC; e++) {
        const float gh = __fmul_rn(g[e], c);
        p[e] = __fsub_rn(__fmul_rn(p[e], keep[e]), __fmul_rn(lr, gh));
    }
}

// The decision of a split step from all-reduced statistics {sum of squares,
// number of ranks that saw a non-finite value}.  One thread.
__global__ void decide_kernel(DevScalars* __restrict__ sc, ScalerArgs sa, const double* __restrict__ stats) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        decide_step(sc, sa, stats[0], stats[1] != 0.0);
        sc->chunk_next = 0;
    }
}

// ---------------------------------------------------------------- host helpers

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool finite(float x) { return std::isfinite(x); }

const char* check_hparams(const neox_hparams* hp) {
    if (!hp) return "hparams is NULL";
    if (!(hp->beta1 >= 0.0f && hp->beta1 < 1.0f)) return "beta1 must be in [0, 1)";
    if (!(hp->beta2 >= 0.0f && hp->beta2 < 1.0f)) return "beta2 must be in [0, 1)";
    if (!(hp->eps >= 0.0f) || !finite(hp->eps)) return "eps must be finite and >= 0";
    if (!finite(hp->clip_norm)) return "clip_norm must be finite";
    if (!(hp->predivide > 0.0f) || !finite(hp->predivide)) return "predivide must be finite and > 0";
    if (!(hp->init_scale > 0.0f) || !finite(hp->init_scale)) return "init_scale must be finite and > 0";
    if (!(hp->scale_factor >= 1.0f) || !finite(hp->scale_factor)) return "scale_factor must be finite and >= 1";
    if (!(hp->min_scale >= 0.0f) || !finite(hp->min_scale)) return "min_scale must be finite and >= 0";
    if (hp->scale_window < 1) return "scale_window must be >= 1";
    if (hp->hysteresis < 0) return "hysteresis must be >= 0";
    if (hp->optimizer != NEOX_ADAMW && hp->optimizer != NEOX_SGD) return "optimizer must be NEOX_ADAMW or NEOX_SGD";
    return nullptr;
}

int hyst_full(const neox_hparams& hp) { return hp.hysteresis > 1 ? hp.hysteresis : 1; }

// The launch arguments of one step over K buffers.  device_bc = false: the
// bias corrections for step t+1 are formed here in double (the step count if
// this step is applied); true: the last pass-1 block forms them on the device.
void make_step_args(const neox_hparams& hp, int K, float lr, long long t, bool device_bc, ScalerArgs& sa,
                    AdamArgs& a) {
    sa = ScalerArgs{};
    sa.post = (double)K / (double)hp.predivide;
    sa.inv_pre = (float)(1.0 / (double)hp.predivide);
    sa.clip = hp.clip_norm;
    sa.factor = hp.scale_factor;
    sa.min_scale = hp.min_scale;
    sa.window = hp.scale_window;
    sa.hyst_full = hyst_full(hp);
    sa.device_bc = device_bc ? 1 : 0;
    sa.lr = lr;
    sa.beta1 = hp.beta1;
    sa.beta2 = hp.beta2;
    a = AdamArgs{};
    a.lr = lr;
    a.b1 = hp.beta1;
    a.b2 = hp.beta2;
    a.omb1 = 1.0f - hp.beta1;
    a.omb2 = 1.0f - hp.beta2;
    a.eps = hp.eps;
    if (!device_bc) {
        const double t1 = (double)(t + 1);
        const double bc1 = 1.0 - std::pow((double)hp.beta1, t1);
        const double bc2 = 1.0 - std::pow((double)hp.beta2, t1);
        a.step_size = (float)((double)lr / bc1);
        a.bcs = (float)std::sqrt(bc2);
    }
    a.device_bc = device_bc ? 1 : 0;
    a.inv_pre = sa.inv_pre;
    a.post = sa.post;
}

int elem_size(neox_dtype) { return 2; }

// Choose the widest vector (8, 4, 2, 1 elements) and a head (peeled, done
// one element per thread) such that every 16-bit array is 2*VEC-byte aligned
// and every FP32 array 16-byte (VEC >= 4) or 4*VEC-byte aligned after it.
// First choice: a head h < 512 that puts every array on a common 1024-,
// 512-, 256- or 128-byte boundary (the coarsest that exists), so that each
// warp's 16-byte accesses cover whole lines and the arrays keep the same
// phase relative to the memory's interleave (arrays that share an element
// offset from 1024-byte boundaries always have one; a 16-byte-only
// alignment left the misaligned 2.57e9-element slice 7% slower).
Layout choose_layout(unsigned long long n, const uintptr_t* a16, int n16, const uintptr_t* a32, int n32, int& vec_out) {
    auto make = [&](int vec, unsigned long long h) {
        Layout L;
        L.n = n;
        L.head = h < n ? h : n;
        L.nvec = (n - L.head) / vec;
        L.tail0 = L.head + L.nvec * vec;
        vec_out = vec;
        return L;
    };
    // The coarsest common boundary first: measured on a 1.41e9-parameter
    // shard at element offset 3, pass 2 ran at 5.76 TB/s with 128-byte
    // alignment, 6.09 with 256 and 6.29 with 1024 (the aligned shard: 6.27).
    for (unsigned al = 1024u; al >= 128u; al >>= 1) {
        for (unsigned h = 0; h < al / 2; h++) {
            bool ok = true;
            for (int i = 0; i < n16 && ok; i++) ok = ((a16[i] + 2u * h) % al) == 0;
            for (int i = 0; i < n32 && ok; i++) ok = ((a32[i] + 4u * h) % al) == 0;
            if (ok) return make(8, h);
        }
    }
    for (int vec = 8; vec >= 1; vec >>= 1) {
        const uintptr_t al16 = 2u * vec;
        const uintptr_t al32 = vec >= 4 ? 16u : 4u * vec;
        for (int h = 0; h < vec; h++) {
            bool ok = true;
            for (int i = 0; i < n16 && ok; i++) ok = ((a16[i] + 2u * h) % al16) == 0;
            for (int i = 0; i < n32 && ok; i++) ok = ((a32[i] + 4u * h) % al32) == 0;
            if (ok) return make(vec, h);
        }
    }
    return make(1, 0);  // unreachable: VEC = 1 always fits
}

// Resident blocks per SM of `kernel` at `threads` per block (no dynamic
// shared memory), cached per kernel: kernels of one signature share a
// function-pointer type, so the cache is keyed by the kernel's address.
template <class K>
int occupancy(K kernel, int threads) {
    static std::mutex mu;
    static std::unordered_map<const void*, int> cache;
    const void* key = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) != cudaSuccess || occ < 1) occ = 1;
    cache.emplace(key, occ);
    return occ;
}

template <class K>
int grid_for(K kernel, int threads, unsigned long long work_items, int sm_count, int cap) {
    const int occ = occupancy(kernel, threads);
    unsigned long long want = (work_items + threads - 1) / threads;
    unsigned long long full = (unsigned long long)sm_count * (unsigned long long)occ;
    unsigned long long g = want < full ? want : full;
    if (g < 1) g = 1;
    if (g > (unsigned long long)cap) g = cap;
    return (int)g;
}

}  // namespace
