// neox_shard.cu -- the per-rank mixed-precision optimizer step over an owned
// flat shard, for NVIDIA B200 (sm_100a).  C ABI in include/neox_shard.h.
//
// Pages followed (title, section):
//  * "GPT-NeoX: how it opened the door to democratised 100B-scale training"
//    (ainews.cool), "技术深度解析" (technical deep-dive): ZeRO stage 1 -- each
//    data-parallel rank updates only the optimizer-state shard it owns.
//  * "OPT: Open Pre-trained Transformer Language Models" (ai-papers.xuzou.cn
//    summary), "计算设置" (compute setup): FP32 Adam state, FP16 weights,
//    dynamic loss scaling; "瓶颈" (bottlenecks): 16 bytes/param of state;
//    "方法适配" (method adaptation): gradient pre-divide, global-norm clip
//    1.0 / 0.3, loss-scaler reset.
//  * AdamW (Loshchilov & Hutter) with bias correction: the pages do not
//    write the update out.
//
// Design (HBM-bound, no dense contraction, so no tensor cores):
//  pass 1  grad_stats_kernel: one streaming read of the K 16-bit gradient
//          buffers with 16-byte vector loads; pre-divide + FP32 sum +
//          unscale in registers; non-finite flag; per-thread sum of squares
//          (FP32 within a vector, FP64 across vectors); warp-shuffle and
//          shared-memory block reduction to per-block partials.  The last
//          block to finish (atomic ticket, no spinning) reduces the partials
//          in a fixed order, so the norm is deterministic, and runs the
//          loss scaler and the clip coefficient on the device.
//  pass 2  adam_kernel: one streaming pass over grad (or the FP32 sum),
//          master, m, v with 16-byte vectors, the blocks taking their work in
//          chunks from a counter that pass 1 zeroed (so SMs that are served
//          faster take more); returns at once when the step overflowed; AdamW
//          with the clip folded in; writes master, m, v and the 16-bit
//          working copy with streaming stores.  sgd_kernel: the same pass
//          with plain SGD, which neither reads nor writes m and v.
// Every FP32 operation of the ingest and of the update uses an explicit
// round-to-nearest intrinsic (no contraction), in the same order as the plain
// definition, so for equal clip coefficients the results are bit-exact with
// a sequential FP32 evaluation.

#include "neox_shard.h"
#include "neox_common.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

namespace {

// The vector loop of pass 1.  KFIX = 1 compiles the single-buffer case with
// K known to be 1; KFIX = 0 takes K at run time.
template <class G, int VEC, bool WRITE_ACC, int KFIX>
__device__ __forceinline__ void pass1_vectors(const GradPtrs& gp, int K_rt, const Layout& L, float inv_pre,
                                              float inv_us, float* __restrict__ acc, double& s, int& bad) {
    const int K = KFIX ? KFIX : K_rt;
    // Several buffers already give several loads in flight per vector: a
    // shorter unroll keeps that variant within its registers.
    constexpr int U = KFIX ? kUnroll1 : 2;
    // Grid-stride over vectors, U strides per iteration (the thread still
    // visits its vectors in the same order, so its sum is unchanged).
    const unsigned long long stride = (unsigned long long)gridDim.x * kThreads1;
    unsigned long long v = (unsigned long long)blockIdx.x * kThreads1 + threadIdx.x;
    if constexpr (KFIX == 1 && VEC == 8 && !WRITE_ACC) {
        // One buffer of 8-element vectors: eight raw 16-byte loads in flight per
        // thread, each vector decoded only when it is summed, so that the raw
        // words (32 registers) and one vector's floats fit the 64 registers of
        // 2 blocks of 512 threads per SM.  Per element the arithmetic is
        // ingest()'s and a thread's vectors are summed in the same order:
        // 1.61 -> 1.46 ms on the 5e9-element BF16 shard (the pass is latency-
        // bound; the loop below keeps four vectors in flight).
        constexpr int U8 = 8;
        const bool pre1 = inv_pre == 1.0f;
        for (; v + (U8 - 1) * stride < L.nvec; v += U8 * stride) {
            uint4 raw[U8];
#pragma unroll
            for (int u = 0; u < U8; u++)
                raw[u] = __ldcs(reinterpret_cast<const uint4*>(gp[0] + L.head + (v + u * stride) * 8));
#pragma unroll
            for (int u = 0; u < U8; u++) {
                const uint32_t wv[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
                float g[8];
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const uint16_t h = uint16_t(wv[e >> 1] >> (16 * (e & 1)));
                    g[e] = __fmul_rn(__fadd_rn(0.0f, pre1 ? G::dec(h) : __fmul_rn(G::dec(h), inv_pre)), inv_us);
                }
                s += vec_sumsq<8>(g, bad);
            }
        }
    }
    for (; v + (U - 1) * stride < L.nvec; v += U * stride) {
        float g[U][VEC];
        if constexpr (KFIX == 1) ingest_batch<G, VEC, U>(gp, K, L.head + v * VEC, stride * VEC, inv_pre, inv_us, g);
        else ingest_batch_pairs<G, VEC, U>(gp, K, L.head + v * VEC, stride * VEC, inv_pre, inv_us, g);
#pragma unroll
        for (int u = 0; u < U; u++) {
            s += vec_sumsq<VEC>(g[u], bad);
            if constexpr (WRITE_ACC) st32<VEC>(acc + L.head + (v + u * stride) * VEC, g[u]);
        }
    }
    for (; v < L.nvec; v += stride) {
        const unsigned long long i = L.head + v * VEC;
        float g[VEC];
        ingest<G, VEC>(gp, K, i, inv_pre, inv_us, g);
        s += vec_sumsq<VEC>(g, bad);
        if constexpr (WRITE_ACC) st32<VEC>(acc + i, g);
    }
}

template <class G, int VEC, bool WRITE_ACC>
__global__ void __launch_bounds__(kThreads1, 1024 / kThreads1)
grad_stats_kernel(GradPtrs gp, int K, Layout L, ScalerArgs sa, float* __restrict__ acc,
                  double* __restrict__ part_s, int* __restrict__ part_b, DevScalars* __restrict__ sc) {
    __shared__ double sh_s[kThreads1 / 32];
    __shared__ int sh_b[kThreads1 / 32];
    __shared__ bool is_last;

    const float inv_us = unscale_factor(sa.post, sc->scale);
    double s = 0.0;
    int bad = 0;

    if (K == 1) pass1_vectors<G, VEC, WRITE_ACC, 1>(gp, K, L, sa.inv_pre, inv_us, acc, s, bad);
    else pass1_vectors<G, VEC, WRITE_ACC, 0>(gp, K, L, sa.inv_pre, inv_us, acc, s, bad);
    if (blockIdx.x == 0) {  // peeled head and ragged tail, one element per thread
        const unsigned long long extra = L.head + (L.n - L.tail0);
        for (unsigned long long j = threadIdx.x; j < extra; j += kThreads1) {
            const unsigned long long i = j < L.head ? j : L.tail0 + (j - L.head);
            float g[1];
            ingest<G, 1>(gp, K, i, sa.inv_pre, inv_us, g);
            s += vec_sumsq<1>(g, bad);
            if constexpr (WRITE_ACC) acc[i] = g[0];
        }
    }

    finish_pass1<kThreads1>(s, bad, part_s, part_b, sc, sa, sh_s, sh_b, &is_last);
}

// ---------------------------------------------------------------- pass 2
struct SegCursor {
    int seg;
    unsigned long long end;
    float keep;  // fl32(1 - fl32(lr * wd)) of segment `seg`
};

__device__ __forceinline__ void seg_seek(SegCursor& c, unsigned long long i, const unsigned long long* seg_end,
                                         const float* seg_wd, int nsegs, float lr) {
    // first segment whose end is > i, searching from the current one
    int lo = c.seg, hi = nsegs - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(seg_end + mid) > i) hi = mid; else lo = mid + 1;
    }
    c.seg = lo;
    c.end = __ldg(seg_end + lo);
    c.keep = __fsub_rn(1.0f, __fmul_rn(lr, __ldg(seg_wd + lo)));
}

// Store the 16-bit cast of p to every extra destination (indexes fixed at
// compile time, so the pointer table stays in registers).
template <class W, int VEC>
__device__ __forceinline__ void store_copies(const WeightCopies& wc, unsigned long long i, const float (&p)[VEC]) {
#pragma unroll
    for (int d = 0; d < kMaxWeightCopies; d++)
        if (d < wc.n) st16<W, VEC>(wc.p[d] + i, p);
}

// The decay factor fl32(1 - fl32(lr * wd)) of each of the VEC elements at i
// (a vector may straddle a segment boundary).  The cursor only moves forward.
template <int VEC>
__device__ __forceinline__ void keep_at(SegCursor& cur, unsigned long long i, const unsigned long long* seg_end,
                                        const float* seg_wd, int nsegs, float lr, float (&keep)[VEC]) {
    if (i >= cur.end) seg_seek(cur, i, seg_end, seg_wd, nsegs, lr);
    if (i + VEC <= cur.end) {
#pragma unroll
        for (int e = 0; e < VEC; e++) keep[e] = cur.keep;
    } else {
#pragma unroll
        for (int e = 0; e < VEC; e++) {
            if (i + e >= cur.end) seg_seek(cur, i + e, seg_end, seg_wd, nsegs, lr);
            keep[e] = cur.keep;
        }
    }
}

// The vector loop of pass 2 (KFIX as in pass1_vectors).
//  AdamW: blocks take chunks of kChunk3 x kThreads3 vectors from a counter in
//    the scalar block (zeroed by pass 1's last block, which this grid waits
//    for).  Blocks whose memory traffic is served faster take more chunks;
//    with the static grid-stride the pass that reads the FP32 sum left its
//    SMs unevenly busy and ran at 5.6 TB/s, against 6.8 with chunks.  Chunks
//    of 2 vectors per thread (64 registers, 4 blocks per SM) measured 6.61
//    TB/s for the 16-bit-gradient form, against 6.25 with chunks of 4 (69
//    registers, 3 blocks per SM) and 6.32 for the static grid-stride.
//    CHUNKED = false (shards of less than one chunk per block, chosen on the
//    host) keeps the static grid-stride: there a chunk's dependent iterations
//    would be the whole latency.
//  SGD: chunks of kUnrollSgd x kThreads3 vectors from the same counter, each
//    thread's kUnrollSgd vectors loaded as one batch (its loads are too few
//    per vector to cover the memory latency one at a time): 6.55 TB/s,
//    against 6.27 for the static grid-stride with the same batches.  Chunks
//    of whole tiles use the AdamW pass's split tiles, all 2U gradient halves
//    loaded as one batch: 6.66 against 6.57 TB/s (468 against 462 Gparams/s
//    for the step); loading the two halves as two batches measured 425.
template <bool SGD, class G, class W, int VEC, bool READ_ACC, int KFIX, bool COPIES, bool CHUNKED>
__device__ __forceinline__ void pass2_vectors(const GradPtrs& gp, int K_rt, const float* __restrict__ acc,
                                              const Layout& L, const AdamArgs& a, float c, float inv_us,
                                              float* __restrict__ master, float* __restrict__ m,
                                              float* __restrict__ v, uint16_t* __restrict__ w,
                                              const unsigned long long* __restrict__ seg_end,
                                              const float* __restrict__ seg_wd, int nsegs, const WeightCopies& wc,
                                              DevScalars* __restrict__ sc) {
    const int K = KFIX ? KFIX : K_rt;
    SegCursor cur{0, 0ull, 1.0f};
    if constexpr (SGD && CHUNKED) {
        // chunks of kUnrollSgd x kThreads3 vectors: each thread's kUnrollSgd
        // vectors of a chunk are loaded as one batch
        constexpr int U = kUnrollSgd;
        constexpr unsigned long long kChunk = (unsigned long long)kThreads3 * U;
        const unsigned long long nchunks = (L.nvec + kChunk - 1) / kChunk;
        __shared__ unsigned int chunk_sh;
        for (;;) {
            if (threadIdx.x == 0) chunk_sh = atomicAdd(&sc->chunk_next, 1u);
            __syncthreads();
            const unsigned long long ch = chunk_sh;
            __syncthreads();                  // chunk_sh is rewritten by the next iteration
            if (ch >= nchunks) break;         // uniform across the block
            if constexpr (VEC == 8 && !READ_ACC) {
                if ((ch + 1) * kChunk <= (L.nvec & ~31ull)) {
                    // the whole chunk in split tiles, the AdamW pass's mapping: lane t
                    // of warp j takes elements 4t + [0, 4) and 128 + 4t + [0, 4) of
                    // tile 32 ch + 8u + j, u = 0..U-1; the 2U gradient halves are
                    // loaded as one batch, then the 2U master halves
                    constexpr unsigned long long kDi = (unsigned long long)kThreads3 * 8;
                    const unsigned long long b0 = L.head + ch * kChunk * 8 + (threadIdx.x >> 5) * 256 +
                                                  (threadIdx.x & 31) * 4;
                    float g[U][8], p[U][8];
                    ingest_halves<G, U>(gp, K, b0, kDi, a.inv_pre, inv_us, g);
#pragma unroll
                    for (int u = 0; u < U; u++) {
                        float lo[4], hi[4];
                        ld32<4>(master + b0 + u * kDi, lo);
                        ld32<4>(master + b0 + u * kDi + 128, hi);
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            p[u][e] = lo[e];
                            p[u][4 + e] = hi[e];
                        }
                    }
#pragma unroll
                    for (int u = 0; u < U; u++) {
                        const unsigned long long i0 = b0 + u * kDi, i1 = i0 + 128;
                        float keep[8], lo[4], hi[4], klo[4], khi[4];
                        keep_at<4>(cur, i0, seg_end, seg_wd, nsegs, a.lr, klo);
                        keep_at<4>(cur, i1, seg_end, seg_wd, nsegs, a.lr, khi);
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            keep[e] = klo[e];
                            keep[4 + e] = khi[e];
                        }
                        sgd_vec<8>(g[u], keep, c, a.lr, p[u]);
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            lo[e] = p[u][e];
                            hi[e] = p[u][4 + e];
                        }
                        st32<4>(master + i0, lo);
                        st32<4>(master + i1, hi);
                        st16<W, 4>(w + i0, lo);
                        st16<W, 4>(w + i1, hi);
                        if constexpr (COPIES) {
                            store_copies<W, 4>(wc, i0, lo);
                            store_copies<W, 4>(wc, i1, hi);
                        }
                    }
                    continue;
                }
            }
            const unsigned long long v0 = ch * kChunk + threadIdx.x;
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; u++) ok[u] = v0 + (unsigned long long)u * kThreads3 < L.nvec;
            float g[U][VEC], p[U][VEC];
            if constexpr (READ_ACC) {
#pragma unroll
                for (int u = 0; u < U; u++)
                    if (ok[u]) ld32<VEC>(acc + L.head + (v0 + (unsigned long long)u * kThreads3) * VEC, g[u]);
            } else {
                ingest_batch_pred<G, VEC, U>(gp, K, L.head + v0 * VEC, (unsigned long long)kThreads3 * VEC, ok,
                                             a.inv_pre, inv_us, g);
            }
#pragma unroll
            for (int u = 0; u < U; u++)
                if (ok[u]) ld32<VEC>(master + L.head + (v0 + (unsigned long long)u * kThreads3) * VEC, p[u]);
#pragma unroll
            for (int u = 0; u < U; u++) {
                if (!ok[u]) continue;
                const unsigned long long i = L.head + (v0 + (unsigned long long)u * kThreads3) * VEC;
                float keep[VEC];
                keep_at<VEC>(cur, i, seg_end, seg_wd, nsegs, a.lr, keep);
                sgd_vec<VEC>(g[u], keep, c, a.lr, p[u]);
                st32<VEC>(master + i, p[u]);
                st16<W, VEC>(w + i, p[u]);
                if constexpr (COPIES) store_copies<W, VEC>(wc, i, p[u]);
            }
        }
    } else if constexpr (SGD) {
        constexpr int U = kUnrollSgd;
        const unsigned long long stride = (unsigned long long)gridDim.x * kThreads3;
        unsigned long long vi = (unsigned long long)blockIdx.x * kThreads3 + threadIdx.x;
        for (; vi + (U - 1) * stride < L.nvec; vi += U * stride) {
            float g[U][VEC], p[U][VEC];
            if constexpr (READ_ACC) {
#pragma unroll
                for (int u = 0; u < U; u++) ld32<VEC>(acc + L.head + (vi + u * stride) * VEC, g[u]);
            } else {
                ingest_batch<G, VEC, U>(gp, K, L.head + vi * VEC, stride * VEC, a.inv_pre, inv_us, g);
            }
#pragma unroll
            for (int u = 0; u < U; u++) ld32<VEC>(master + L.head + (vi + u * stride) * VEC, p[u]);
#pragma unroll
            for (int u = 0; u < U; u++) {
                const unsigned long long i = L.head + (vi + u * stride) * VEC;
                float keep[VEC];
                keep_at<VEC>(cur, i, seg_end, seg_wd, nsegs, a.lr, keep);
                sgd_vec<VEC>(g[u], keep, c, a.lr, p[u]);
                st32<VEC>(master + i, p[u]);
                st16<W, VEC>(w + i, p[u]);
                if constexpr (COPIES) store_copies<W, VEC>(wc, i, p[u]);
            }
        }
        for (; vi < L.nvec; vi += stride) {
            const unsigned long long i = L.head + vi * VEC;
            float g[VEC], p[VEC], keep[VEC];
            if constexpr (READ_ACC) ld32<VEC>(acc + i, g);
            else ingest<G, VEC>(gp, K, i, a.inv_pre, inv_us, g);
            ld32<VEC>(master + i, p);
            keep_at<VEC>(cur, i, seg_end, seg_wd, nsegs, a.lr, keep);
            sgd_vec<VEC>(g, keep, c, a.lr, p);
            st32<VEC>(master + i, p);
            st16<W, VEC>(w + i, p);
            if constexpr (COPIES) store_copies<W, VEC>(wc, i, p);
        }
    } else if constexpr (!CHUNKED) {
        const unsigned long long stride = (unsigned long long)gridDim.x * kThreads3;
        for (unsigned long long vi = (unsigned long long)blockIdx.x * kThreads3 + threadIdx.x; vi < L.nvec;
             vi += stride) {
            const unsigned long long i = L.head + vi * VEC;
            float g[VEC], p[VEC], mm[VEC], vv[VEC], keep[VEC];
            if constexpr (READ_ACC) ld32<VEC>(acc + i, g);
            else ingest<G, VEC>(gp, K, i, a.inv_pre, inv_us, g);
            ld32<VEC>(master + i, p);
            ld32<VEC>(m + i, mm);
            ld32<VEC>(v + i, vv);
            keep_at<VEC>(cur, i, seg_end, seg_wd, nsegs, a.lr, keep);
            adam_vec<VEC>(g, keep, c, a, p, mm, vv);
            st32<VEC>(master + i, p);
            st32<VEC>(m + i, mm);
            st32<VEC>(v + i, vv);
            st16<W, VEC>(w + i, p);
            if constexpr (COPIES) store_copies<W, VEC>(wc, i, p);
        }
    } else {
        constexpr unsigned long long kChunk = (unsigned long long)kThreads3 * kChunk3;
        const unsigned long long nchunks = (L.nvec + kChunk - 1) / kChunk;
        // Vectors of whole 32-vector tiles (VEC = 8) are split: lane t of tile w
        // takes elements 256w + 4t + [0, 4) and 256w + 128 + 4t + [0, 4), so
        // each warp-wide 16-byte FP32 access covers 512 contiguous bytes (16
        // sectors, all used).  Eight consecutive elements per lane make every
        // FP32 access a 32-byte stride of 16-byte pieces: 32 sectors per
        // request, each half used, twice the L1-L2 sectors of the data.  The
        // split took the pass from 6.61 to 6.81 TB/s on the Pythia-shaped
        // shard and from 6.44 to 6.80 on the 5e9-element BF16 shard.
        const unsigned long long nsplit = L.nvec & ~31ull;
        __shared__ unsigned int chunk_sh;
        for (;;) {
            if (threadIdx.x == 0) chunk_sh = atomicAdd(&sc->chunk_next, 1u);
            __syncthreads();
            const unsigned long long ch = chunk_sh;
            __syncthreads();                  // chunk_sh is rewritten by the next iteration
            if (ch >= nchunks) break;         // uniform across the block
            for (int k = 0; k < kChunk3; k++) {
                const unsigned long long vi = ch * kChunk + (unsigned long long)k * kThreads3 + threadIdx.x;
                if (vi >= L.nvec) break;
                if constexpr (VEC == 8) {
                    if (vi < nsplit) {
                        const unsigned long long i0 = L.head + (vi >> 5) * 256 + (vi & 31) * 4, i1 = i0 + 128;
                        float g0[4], g1[4], p0[4], p1[4], m0[4], m1[4], v0[4], v1[4], k0[4], k1[4];
                        if constexpr (READ_ACC) {
                            ld32<4>(acc + i0, g0);
                            ld32<4>(acc + i1, g1);
                        } else {
                            ingest<G, 4>(gp, K, i0, a.inv_pre, inv_us, g0);
                            ingest<G, 4>(gp, K, i1, a.inv_pre, inv_us, g1);
                        }
                        ld32<4>(master + i0, p0);
                        ld32<4>(master + i1, p1);
                        ld32<4>(m + i0, m0);
                        ld32<4>(m + i1, m1);
                        ld32<4>(v + i0, v0);
                        ld32<4>(v + i1, v1);
                        keep_at<4>(cur, i0, seg_end, seg_wd, nsegs, a.lr, k0);
                        keep_at<4>(cur, i1, seg_end, seg_wd, nsegs, a.lr, k1);
                        adam_vec<4>(g0, k0, c, a, p0, m0, v0);
                        adam_vec<4>(g1, k1, c, a, p1, m1, v1);
                        st32<4>(master + i0, p0);
                        st32<4>(master + i1, p1);
                        st32<4>(m + i0, m0);
                        st32<4>(m + i1, m1);
                        st32<4>(v + i0, v0);
                        st32<4>(v + i1, v1);
                        st16<W, 4>(w + i0, p0);
                        st16<W, 4>(w + i1, p1);
                        if constexpr (COPIES) {
                            store_copies<W, 4>(wc, i0, p0);
                            store_copies<W, 4>(wc, i1, p1);
                        }
                        continue;
                    }
                }
                // contiguous mapping (VEC < 8, or past the whole tiles, which cover
                // elements head .. head + 8 nsplit - 1)
                const unsigned long long i = L.head + vi * VEC;
                float g[VEC], p[VEC], mm[VEC], vv[VEC], keep[VEC];
                if constexpr (READ_ACC) ld32<VEC>(acc + i, g);
                else ingest<G, VEC>(gp, K, i, a.inv_pre, inv_us, g);
                ld32<VEC>(master + i, p);
                ld32<VEC>(m + i, mm);
                ld32<VEC>(v + i, vv);
                keep_at<VEC>(cur, i, seg_end, seg_wd, nsegs, a.lr, keep);
                adam_vec<VEC>(g, keep, c, a, p, mm, vv);
                st32<VEC>(master + i, p);
                st32<VEC>(m + i, mm);
                st32<VEC>(v + i, vv);
                st16<W, VEC>(w + i, p);
                if constexpr (COPIES) store_copies<W, VEC>(wc, i, p);
            }
        }
    }
}

// The whole of pass 2 for one grid: the vector loop, then (block 0) the
// peeled head and the ragged tail one element per thread.
template <bool SGD, class G, class W, int VEC, bool READ_ACC, bool COPIES, bool CHUNKED>
__device__ __forceinline__ void update_shard(const GradPtrs& gp, int K, const float* __restrict__ acc,
                                             const Layout& L, const AdamArgs& a_arg, float* __restrict__ master,
                                             float* __restrict__ m, float* __restrict__ v, uint16_t* __restrict__ w,
                                             const unsigned long long* __restrict__ seg_end,
                                             const float* __restrict__ seg_wd, int nsegs,
                                             DevScalars* __restrict__ sc, const WeightCopies& wc) {
    // Programmatic dependent launch: everything below reads what pass 1 wrote.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (sc->overflow) return;  // skipped step: nothing is written
    const float c = sc->coef;
    AdamArgs a = a_arg;
    const float inv_us = unscale_factor(a.post, sc->scale_used);
    if (a.device_bc) {
        a.lr = sc->lr;
        a.step_size = sc->step_size;
        a.bcs = sc->bc2_sqrt;
    }

    if (K == 1)
        pass2_vectors<SGD, G, W, VEC, READ_ACC, 1, COPIES, CHUNKED>(gp, K, acc, L, a, c, inv_us, master, m, v, w, seg_end, seg_wd,
                                                           nsegs, wc, sc);
    else
        pass2_vectors<SGD, G, W, VEC, READ_ACC, 0, COPIES, CHUNKED>(gp, K, acc, L, a, c, inv_us, master, m, v, w, seg_end, seg_wd,
                                                           nsegs, wc, sc);
    if (blockIdx.x == 0) {
        const unsigned long long extra = L.head + (L.n - L.tail0);
        for (unsigned long long j = threadIdx.x; j < extra; j += kThreads3) {
            const unsigned long long i = j < L.head ? j : L.tail0 + (j - L.head);
            float g[1], p[1] = {master[i]}, keep[1];
            if constexpr (READ_ACC) g[0] = acc[i];
            else ingest<G, 1>(gp, K, i, a.inv_pre, inv_us, g);
            SegCursor c1{0, 0ull, 1.0f};
            seg_seek(c1, i, seg_end, seg_wd, nsegs, a.lr);
            keep[0] = c1.keep;
            if constexpr (SGD) {
                sgd_vec<1>(g, keep, c, a.lr, p);
            } else {
                float mm[1] = {m[i]}, vv[1] = {v[i]};
                adam_vec<1>(g, keep, c, a, p, mm, vv);
                m[i] = mm[0];
                v[i] = vv[0];
            }
            master[i] = p[0];
            w[i] = W::enc(p[0]);
            if constexpr (COPIES) store_copies<W, 1>(wc, i, p);
        }
    }
}

// Pass 2 with AdamW.
template <class G, class W, int VEC, bool READ_ACC, bool COPIES, bool CHUNKED>
__global__ void __launch_bounds__(kThreads3)
adam_kernel(GradPtrs gp, int K, const float* __restrict__ acc, Layout L, AdamArgs a,
            float* __restrict__ master, float* __restrict__ m, float* __restrict__ v, uint16_t* __restrict__ w,
            const unsigned long long* __restrict__ seg_end, const float* __restrict__ seg_wd, int nsegs,
            DevScalars* __restrict__ sc, WeightCopies wc) {
    update_shard<false, G, W, VEC, READ_ACC, COPIES, CHUNKED>(gp, K, acc, L, a, master, m, v, w, seg_end, seg_wd, nsegs,
                                                              sc, wc);
}

// Pass 2 with plain SGD (m and v are not touched).
template <class G, class W, int VEC, bool READ_ACC, bool COPIES, bool CHUNKED>
__global__ void __launch_bounds__(kThreads3)
sgd_kernel(GradPtrs gp, int K, const float* __restrict__ acc, Layout L, AdamArgs a,
           float* __restrict__ master, float* __restrict__ m, float* __restrict__ v, uint16_t* __restrict__ w,
           const unsigned long long* __restrict__ seg_end, const float* __restrict__ seg_wd, int nsegs,
           DevScalars* __restrict__ sc, WeightCopies wc) {
    update_shard<true, G, W, VEC, READ_ACC, COPIES, CHUNKED>(gp, K, acc, L, a, master, m, v, w, seg_end, seg_wd, nsegs,
                                                             sc, wc);
}

}  // namespace

// ====================================================================== host

constexpr unsigned long long kAccPad = 256;  // floats of slack: the buffer is shifted by up to 1 KB

struct neox_shard {
    int device = 0;
    int sm_count = 0;
    unsigned long long numel = 0;
    neox_dtype wdtype = NEOX_FP16, gdtype = NEOX_FP16;
    float* master = nullptr;
    float* m = nullptr;
    float* v = nullptr;
    neox_hparams hp{};
    int max_grads = 1;
    bool accumulate = false;          // NEOX_SHARD_ACCUMULATE: the FP32 sum buffer at every K
    // mirrors of the device scaler state (refreshed after every step)
    float scale = 1.0f;
    int32_t good = 0;
    long long t = 0;
    // owned device memory
    DevScalars* d_sc = nullptr;
    double* d_part_s = nullptr;
    int* d_part_b = nullptr;
    int max_parts = 0;
    unsigned long long* d_seg_end = nullptr;
    float* d_seg_wd = nullptr;
    int nsegs = 0;
    float* d_acc = nullptr;  // FP32 sum of the K buffers (numel + kAccPad floats)
    DevScalars* h_sc = nullptr;  // pinned result slot
    unsigned long long owned_bytes = 0;
    // profiling
    bool profiling = false;
    bool async_used = false;          // an asynchronous step was issued (replays may follow)
    WeightCopies wcopies{};           // extra destinations of the working weights
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
    neox_profile prof{};
    std::string last_error;
};

namespace {

thread_local std::string g_create_error;

neox_status fail(neox_shard* h, neox_status st, const std::string& msg) {
    if (h) h->last_error = msg; else g_create_error = msg;
    return st;
}

neox_status cuda_fail(neox_shard* h, cudaError_t e, const char* what) {
    std::string msg = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return fail(h, e == cudaErrorMemoryAllocation ? NEOX_ERR_OUT_OF_MEMORY : NEOX_ERR_CUDA, msg);
}

template <class G, int VEC, bool ACC>
cudaError_t launch_pass1(neox_shard* h, const GradPtrs& gp, int K, const Layout& L, const ScalerArgs& sa,
                         float* acc, cudaStream_t st) {
    auto kern = grad_stats_kernel<G, VEC, ACC>;
    const int grid = grid_for(kern, kThreads1, L.nvec, h->sm_count, h->max_parts);
    kern<<<grid, kThreads1, 0, st>>>(gp, K, L, sa, acc, h->d_part_s, h->d_part_b, h->d_sc);
    return cudaGetLastError();
}

template <class G, class W, int VEC, bool ACC>
cudaError_t launch_pass2(neox_shard* h, const GradPtrs& gp, int K, const float* acc, const Layout& L,
                         const AdamArgs& a, uint16_t* w, cudaStream_t st) {
    const bool sgd = h->hp.optimizer == NEOX_SGD, copies = h->wcopies.n > 0;
    auto kern = sgd ? (copies ? sgd_kernel<G, W, VEC, ACC, true, true> : sgd_kernel<G, W, VEC, ACC, false, true>)
                    : (copies ? adam_kernel<G, W, VEC, ACC, true, true> : adam_kernel<G, W, VEC, ACC, false, true>);
    int grid = grid_for(kern, kThreads3, L.nvec, h->sm_count, 1 << 20);
    // Chunks only when the shard has at least one per block; the grid-stride
    // instance has its own occupancy, hence its own grid
    if (L.nvec < (unsigned long long)grid * kThreads3 * (sgd ? kUnrollSgd : kChunk3)) {
        kern = sgd ? (copies ? sgd_kernel<G, W, VEC, ACC, true, false> : sgd_kernel<G, W, VEC, ACC, false, false>)
                   : (copies ? adam_kernel<G, W, VEC, ACC, true, false> : adam_kernel<G, W, VEC, ACC, false, false>);
        grid = grid_for(kern, kThreads3, L.nvec, h->sm_count, 1 << 20);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads3);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float* accp = acc;
    const unsigned long long* se = h->d_seg_end;
    const float* sw = h->d_seg_wd;
    DevScalars* sc = h->d_sc;
    return cudaLaunchKernelEx(&cfg, kern, gp, K, accp, L, a, h->master, h->m, h->v, w, se, sw, h->nsegs, sc,
                              h->wcopies);
}

template <class G, int VEC>
cudaError_t dispatch1(neox_shard* h, const GradPtrs& gp, int K, const Layout& L, const ScalerArgs& sa,
                      float* acc, cudaStream_t st) {
    return acc ? launch_pass1<G, VEC, true>(h, gp, K, L, sa, acc, st)
               : launch_pass1<G, VEC, false>(h, gp, K, L, sa, acc, st);
}

template <class G>
cudaError_t dispatch1v(neox_shard* h, int vec, const GradPtrs& gp, int K, const Layout& L, const ScalerArgs& sa,
                       float* acc, cudaStream_t st) {
    switch (vec) {
        case 8: return dispatch1<G, 8>(h, gp, K, L, sa, acc, st);
        case 4: return dispatch1<G, 4>(h, gp, K, L, sa, acc, st);
        case 2: return dispatch1<G, 2>(h, gp, K, L, sa, acc, st);
        default: return dispatch1<G, 1>(h, gp, K, L, sa, acc, st);
    }
}

template <class G, class W, int VEC>
cudaError_t dispatch2(neox_shard* h, const GradPtrs& gp, int K, const float* acc, const Layout& L,
                      const AdamArgs& a, uint16_t* w, cudaStream_t st) {
    return acc ? launch_pass2<G, W, VEC, true>(h, gp, K, acc, L, a, w, st)
               : launch_pass2<G, W, VEC, false>(h, gp, K, acc, L, a, w, st);
}

template <class G, class W>
cudaError_t dispatch2v(neox_shard* h, int vec, const GradPtrs& gp, int K, const float* acc, const Layout& L,
                       const AdamArgs& a, uint16_t* w, cudaStream_t st) {
    switch (vec) {
        case 8: return dispatch2<G, W, 8>(h, gp, K, acc, L, a, w, st);
        case 4: return dispatch2<G, W, 4>(h, gp, K, acc, L, a, w, st);
        case 2: return dispatch2<G, W, 2>(h, gp, K, acc, L, a, w, st);
        default: return dispatch2<G, W, 1>(h, gp, K, acc, L, a, w, st);
    }
}

void free_all(neox_shard* h) {
    if (h->d_sc) cudaFree(h->d_sc);
    if (h->d_part_s) cudaFree(h->d_part_s);
    if (h->d_part_b) cudaFree(h->d_part_b);
    if (h->d_seg_end) cudaFree(h->d_seg_end);
    if (h->d_seg_wd) cudaFree(h->d_seg_wd);
    if (h->d_acc) cudaFree(h->d_acc);
    if (h->h_sc) cudaFreeHost(h->h_sc);
    for (auto& e : h->ev)
        if (e) cudaEventDestroy(e);
}

// Bring the host copy of the scaler state up to date.  Once asynchronous
// steps were issued (possibly replayed from a CUDA graph, which this library
// does not see), the device copy is the only current one: wait for the device
// and read it.
neox_status refresh_mirror(neox_shard* h) {
    if (!h->async_used) return NEOX_OK;
    DeviceGuard g(h->device);
    cudaError_t e;
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(h, e, "waiting for asynchronous steps");
    DevScalars r;
    if ((e = cudaMemcpy(&r, h->d_sc, sizeof(r), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(h, e, "reading the device scaler state");
    h->scale = r.scale;
    h->good = r.good;
    h->t = r.t;
    return NEOX_OK;
}

// Validate the arguments of a step and enqueue its two kernels on `st`.
// device_bc = false: bias corrections from the host copy of t (synchronous
// steps, whose caller keeps that copy current).  device_bc = true: the last
// pass-1 block forms them from the device step count and writes `result`.
// timed: record the profiling events around the two launches.
enum StepMode { kFused = 0, kStatsOnly = 1, kApply = 2 };

neox_status enqueue_step(neox_shard* h, const void* const* grads, int32_t num_grads, void* params, float lr,
                         const float* lr_dev, cudaStream_t st, bool device_bc, neox_step_result* result,
                         bool timed, StepMode mode = kFused, double* stats = nullptr) {
    if (num_grads < 1 || num_grads > kMaxGrads) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "num_grads must be in [1, 64]");
    if (!grads) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "grads is NULL");
    if (!lr_dev && (!finite(lr) || lr < 0.0f)) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "lr must be finite and >= 0");
    GradPtrs gp{};
    uintptr_t a16[kMaxGrads + 1 + kMaxWeightCopies];
    if (h->numel > 0) {
        if (!params) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "params is NULL");
        if ((uintptr_t)params & 1u) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "params must be 2-byte aligned");
        for (int k = 0; k < num_grads; k++) {
            if (!grads[k]) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "grads[" + std::to_string(k) + "] is NULL");
            if ((uintptr_t)grads[k] & 1u)
                return fail(h, NEOX_ERR_INVALID_ARGUMENT, "grads[" + std::to_string(k) + "] must be 2-byte aligned");
            gp.p[k] = static_cast<const uint16_t*>(grads[k]);
            a16[k] = (uintptr_t)grads[k];
        }
        a16[num_grads] = (uintptr_t)params;
        for (int d = 0; d < h->wcopies.n; d++) a16[num_grads + 1 + d] = (uintptr_t)h->wcopies.p[d];
    }
    if (result && ((uintptr_t)result & 7u)) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "result must be 8-byte aligned");
    if (mode != kFused && (!stats || ((uintptr_t)stats & 7u)))
        return fail(h, NEOX_ERR_INVALID_ARGUMENT, "stats must be a non-NULL, 8-byte aligned device pointer");
    if (lr_dev && ((uintptr_t)lr_dev & 3u)) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "lr_device must be 4-byte aligned");

    const bool use_acc = h->d_acc != nullptr && (num_grads >= 5 || h->accumulate);
    uintptr_t a32[3] = {(uintptr_t)h->master, (uintptr_t)h->m, (uintptr_t)h->v};
    int vec = 1;
    Layout L = h->numel > 0 ? choose_layout(h->numel, a16, num_grads + 1 + h->wcopies.n, a32, 3, vec)
                            : Layout{0, 0, 0, 0};
    float* acc = nullptr;
    if (use_acc) {  // shift the buffer so that &acc[head] sits on a 1024-byte boundary, like the other arrays
        const uintptr_t a = (uintptr_t)(h->d_acc + L.head);
        acc = h->d_acc + ((1024u - a % 1024u) % 1024u) / sizeof(float);
    }

    ScalerArgs sa;
    AdamArgs a;
    make_step_args(h->hp, num_grads, lr, h->t, device_bc, sa, a);
    sa.lr_ptr = lr_dev;
    sa.result = result;
    sa.stats_out = mode == kStatsOnly ? stats : nullptr;

    cudaError_t e;
    if (timed && (e = cudaEventRecord(h->ev[0], st)) != cudaSuccess) return cuda_fail(h, e, "cudaEventRecord");
    if (mode == kApply) {  // the decision from the all-reduced statistics
        decide_kernel<<<1, 1, 0, st>>>(h->d_sc, sa, stats);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(h, e, "decision launch");
    } else {
        if (h->gdtype == NEOX_FP16) e = dispatch1v<F16>(h, vec, gp, num_grads, L, sa, acc, st);
        else e = dispatch1v<BF16>(h, vec, gp, num_grads, L, sa, acc, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "pass-1 launch");
    }
    h->prof.launches += 1;
    if (timed && (e = cudaEventRecord(h->ev[1], st)) != cudaSuccess) return cuda_fail(h, e, "cudaEventRecord");
    if (h->numel > 0 && mode != kStatsOnly) {
        uint16_t* w = static_cast<uint16_t*>(params);
        if (h->gdtype == NEOX_FP16) {
            e = h->wdtype == NEOX_FP16 ? dispatch2v<F16, F16>(h, vec, gp, num_grads, acc, L, a, w, st)
                                       : dispatch2v<F16, BF16>(h, vec, gp, num_grads, acc, L, a, w, st);
        } else {
            e = h->wdtype == NEOX_FP16 ? dispatch2v<BF16, F16>(h, vec, gp, num_grads, acc, L, a, w, st)
                                       : dispatch2v<BF16, BF16>(h, vec, gp, num_grads, acc, L, a, w, st);
        }
        if (e != cudaSuccess) return cuda_fail(h, e, "pass-2 launch");
        h->prof.launches += 1;
    }
    if (timed && (e = cudaEventRecord(h->ev[2], st)) != cudaSuccess) return cuda_fail(h, e, "cudaEventRecord");
    return NEOX_OK;
}

// Wait for the step on `st`, read its scalar block, fill `out`, refresh the
// host copy of the scaler state and account the profiling events.
neox_status read_result(neox_shard* h, cudaStream_t st, neox_step_result* out) {
    cudaError_t e;
    if ((e = cudaMemcpyAsync(h->h_sc, h->d_sc, sizeof(DevScalars), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return cuda_fail(h, e, "cudaMemcpyAsync result");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(h, e, "step execution");
    const DevScalars& r = *h->h_sc;
    out->overflow = r.overflow;
    out->grad_norm = r.norm;
    out->clip_coef = r.coef;
    out->loss_scale = r.scale_used;
    out->loss_scale_next = r.scale;
    out->good_steps = r.good;
    out->applied_steps = r.t;
    h->scale = r.scale;
    h->good = r.good;
    h->t = r.t;
    if (h->profiling) {
        float t01 = 0.f, t12 = 0.f;
        cudaEventElapsedTime(&t01, h->ev[0], h->ev[1]);
        cudaEventElapsedTime(&t12, h->ev[1], h->ev[2]);
        h->prof.steps += 1;
        h->prof.grad_pass_ms += t01;
        h->prof.update_pass_ms += t12;
        h->prof.last_grad_pass_ms = t01;
        h->prof.last_update_pass_ms = t12;
    }
    return NEOX_OK;
}

}  // namespace

extern "C" {

const char* neox_status_string(neox_status s) {
    switch (s) {
        case NEOX_OK: return "ok";
        case NEOX_ERR_INVALID_ARGUMENT: return "invalid argument";
        case NEOX_ERR_CUDA: return "CUDA error";
        case NEOX_ERR_OUT_OF_MEMORY: return "out of memory";
        case NEOX_ERR_UNSUPPORTED: return "unsupported";
    }
    return "unknown status";
}

const char* neox_last_error(const neox_shard* h) {
    return h ? h->last_error.c_str() : g_create_error.c_str();
}

uint64_t neox_model_state_bytes(uint64_t numel, neox_dtype wdtype, neox_dtype gdtype) {
    return numel * (uint64_t)(elem_size(wdtype) + elem_size(gdtype) + 3 * (int)sizeof(float));
}

uint64_t neox_shard_scratch_bytes(const neox_shard* h) { return h ? h->owned_bytes : 0; }

neox_status neox_shard_create(const neox_shard_desc* d, const neox_hparams* hp, int device, neox_shard** out) {
    g_create_error.clear();
    if (!out) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "out is NULL");
    if (!d) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "desc is NULL");
    if (const char* why = check_hparams(hp)) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, why);
    if ((d->wdtype != NEOX_FP16 && d->wdtype != NEOX_BF16) || (d->gdtype != NEOX_FP16 && d->gdtype != NEOX_BF16))
        return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "dtype must be NEOX_FP16 or NEOX_BF16");
    if (d->max_grads < 0 || d->max_grads > kMaxGrads)
        return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "max_grads must be in [0, 64]");
    if (d->flags & ~NEOX_SHARD_ACCUMULATE) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "unknown flags");
    if (d->numel > 0) {
        if (!d->master || !d->exp_avg || !d->exp_avg_sq)
            return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "master/exp_avg/exp_avg_sq must be non-NULL");
        if (((uintptr_t)d->master | (uintptr_t)d->exp_avg | (uintptr_t)d->exp_avg_sq) & 3u)
            return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "FP32 state arrays must be 4-byte aligned");
    }
    if (!finite(d->default_weight_decay)) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "weight decay must be finite");
    // segment table -> (end, wd) arrays
    int nsegs = 1;
    unsigned long long* ends = nullptr;
    float* wds = nullptr;
    if (d->segs) {
        if (d->nsegs < 1) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "nsegs must be >= 1 with a table");
        nsegs = d->nsegs;
        unsigned long long pos = 0;
        for (int i = 0; i < nsegs; i++) {
            const neox_segment& s = d->segs[i];
            if (s.offset != pos || s.numel == 0)
                return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT,
                            "segments must be sorted, non-empty and tile [0, numel) (segment " + std::to_string(i) + ")");
            if (!finite(s.weight_decay))
                return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "segment weight decay must be finite");
            pos += s.numel;
        }
        if (pos != d->numel) return fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "segments do not cover numel");
    }
    ends = new (std::nothrow) unsigned long long[nsegs];
    wds = new (std::nothrow) float[nsegs];
    if (!ends || !wds) {
        delete[] ends;
        delete[] wds;
        return fail(nullptr, NEOX_ERR_OUT_OF_MEMORY, "host allocation failed");
    }
    if (d->segs) {
        for (int i = 0; i < nsegs; i++) { ends[i] = d->segs[i].offset + d->segs[i].numel; wds[i] = d->segs[i].weight_decay; }
    } else {
        ends[0] = d->numel;
        wds[0] = d->default_weight_decay;
    }

    auto* h = new (std::nothrow) neox_shard();
    if (!h) { delete[] ends; delete[] wds; return fail(nullptr, NEOX_ERR_OUT_OF_MEMORY, "host allocation failed"); }
    h->device = device;
    h->numel = d->numel;
    h->wdtype = d->wdtype;
    h->gdtype = d->gdtype;
    h->master = d->master;
    h->m = d->exp_avg;
    h->v = d->exp_avg_sq;
    h->hp = *hp;
    h->max_grads = d->max_grads < 1 ? 1 : d->max_grads;
    h->accumulate = (d->flags & NEOX_SHARD_ACCUMULATE) != 0;
    h->scale = hp->init_scale;
    h->nsegs = nsegs;

    neox_status st = NEOX_OK;
    cudaError_t e;
    {
        int ndev = 0;
        if ((e = cudaGetDeviceCount(&ndev)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaGetDeviceCount"); goto done; }
        if (device < 0 || device >= ndev) { st = fail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "no such CUDA device"); goto done; }
        DeviceGuard g(device);
        if (!g.ok) { st = fail(nullptr, NEOX_ERR_CUDA, "cudaSetDevice failed"); goto done; }
        cudaDeviceProp prop;
        if ((e = cudaGetDeviceProperties(&prop, device)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaGetDeviceProperties"); goto done; }
        if (prop.major != 10) { st = fail(nullptr, NEOX_ERR_UNSUPPORTED, "this library is built for sm_100a (B200)"); goto done; }
        h->sm_count = prop.multiProcessorCount;
        h->max_parts = h->sm_count * kMaxBlocksPerSm;
        size_t bytes;
        if ((e = cudaMalloc(&h->d_sc, sizeof(DevScalars))) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMalloc scalars"); goto done; }
        bytes = sizeof(DevScalars);
        if ((e = cudaMalloc(&h->d_part_s, sizeof(double) * h->max_parts)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMalloc partials"); goto done; }
        if ((e = cudaMalloc(&h->d_part_b, sizeof(int) * h->max_parts)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMalloc partials"); goto done; }
        bytes += (sizeof(double) + sizeof(int)) * h->max_parts;
        if ((e = cudaMalloc(&h->d_seg_end, sizeof(unsigned long long) * nsegs)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMalloc segments"); goto done; }
        if ((e = cudaMalloc(&h->d_seg_wd, sizeof(float) * nsegs)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMalloc segments"); goto done; }
        bytes += (sizeof(unsigned long long) + sizeof(float)) * nsegs;
        if ((h->max_grads >= 5 || h->accumulate) && h->numel > 0) {
            if ((e = cudaMalloc(&h->d_acc, sizeof(float) * (h->numel + kAccPad))) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMalloc accumulation buffer"); goto done; }
            bytes += sizeof(float) * (h->numel + kAccPad);
        }
        h->owned_bytes = bytes;
        if ((e = cudaMallocHost(&h->h_sc, sizeof(DevScalars))) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMallocHost"); goto done; }
        for (auto& ev : h->ev)
            if ((e = cudaEventCreate(&ev)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaEventCreate"); goto done; }
        if ((e = cudaMemcpy(h->d_seg_end, ends, sizeof(unsigned long long) * nsegs, cudaMemcpyHostToDevice)) != cudaSuccess ||
            (e = cudaMemcpy(h->d_seg_wd, wds, sizeof(float) * nsegs, cudaMemcpyHostToDevice)) != cudaSuccess) {
            st = cuda_fail(nullptr, e, "cudaMemcpy segments");
            goto done;
        }
        DevScalars init{};
        init.scale = hp->init_scale;
        init.scale_used = hp->init_scale;
        init.hyst = hyst_full(*hp);
        if ((e = cudaMemcpy(h->d_sc, &init, sizeof(init), cudaMemcpyHostToDevice)) != cudaSuccess) { st = cuda_fail(nullptr, e, "cudaMemcpy scalars"); goto done; }
    }
done:
    delete[] ends;
    delete[] wds;
    if (st != NEOX_OK) {
        DeviceGuard g(device);
        free_all(h);
        delete h;
        return st;
    }
    *out = h;
    return NEOX_OK;
}

void neox_shard_destroy(neox_shard* h) {
    if (!h) return;
    {
        DeviceGuard g(h->device);
        free_all(h);
    }
    delete h;
}

neox_status neox_shard_set_hparams(neox_shard* h, const neox_hparams* hp) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (const char* why = check_hparams(hp)) return fail(h, NEOX_ERR_INVALID_ARGUMENT, why);
    h->hp = *hp;
    return NEOX_OK;
}

neox_status neox_shard_set_weight_copies(neox_shard* h, void* const* dsts, int32_t n) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (n < 0 || n > kMaxWeightCopies) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "n must be in [0, 8]");
    if (n > 0 && !dsts) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "dsts is NULL");
    WeightCopies wc{};
    for (int d = 0; d < n; d++) {
        if (!dsts[d] || ((uintptr_t)dsts[d] & 1u))
            return fail(h, NEOX_ERR_INVALID_ARGUMENT, "weight copy " + std::to_string(d) + " NULL or not 2-byte aligned");
        wc.p[d] = static_cast<uint16_t*>(dsts[d]);
    }
    wc.n = n;
    h->wcopies = wc;
    return NEOX_OK;
}

neox_status neox_shard_get_state(const neox_shard* h, float* scale, int32_t* good, int64_t* t) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (neox_status s = refresh_mirror(const_cast<neox_shard*>(h)); s != NEOX_OK) return s;
    if (scale) *scale = h->scale;
    if (good) *good = h->good;
    if (t) *t = h->t;
    return NEOX_OK;
}

neox_status neox_shard_set_state(neox_shard* h, float scale, int32_t good, int64_t t) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.0f) || !finite(scale) || good < 0 || t < 0)
        return fail(h, NEOX_ERR_INVALID_ARGUMENT, "state needs a finite scale > 0, good >= 0, t >= 0");
    DeviceGuard g(h->device);
    if (h->async_used) {
        cudaError_t e0 = cudaDeviceSynchronize();
        if (e0 != cudaSuccess) return cuda_fail(h, e0, "waiting for asynchronous steps");
    }
    DevScalars s{};
    s.scale = scale;
    s.scale_used = scale;
    s.good = good;
    s.t = t;
    s.hyst = hyst_full(h->hp);
    cudaError_t e = cudaMemcpy(h->d_sc, &s, sizeof(s), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemcpy scalars");
    h->scale = scale;
    h->good = good;
    h->t = t;
    return NEOX_OK;
}

neox_status neox_shard_get_hysteresis(const neox_shard* h, int32_t* count) {
    if (!h || !count) return NEOX_ERR_INVALID_ARGUMENT;
    auto* hm = const_cast<neox_shard*>(h);
    DeviceGuard g(h->device);
    cudaError_t e = h->async_used ? cudaDeviceSynchronize() : cudaSuccess;
    if (e == cudaSuccess) e = cudaMemcpy(count, &h->d_sc->hyst, sizeof(int32_t), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? NEOX_OK : cuda_fail(hm, e, "reading the hysteresis count");
}

neox_status neox_shard_set_hysteresis(neox_shard* h, int32_t count) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (count < 0) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "the hysteresis count must be >= 0");
    DeviceGuard g(h->device);
    cudaError_t e = h->async_used ? cudaDeviceSynchronize() : cudaSuccess;
    if (e == cudaSuccess) e = cudaMemcpy(&h->d_sc->hyst, &count, sizeof(int32_t), cudaMemcpyHostToDevice);
    return e == cudaSuccess ? NEOX_OK : cuda_fail(h, e, "writing the hysteresis count");
}

neox_status neox_shard_set_profiling(neox_shard* h, int32_t enable) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->profiling = enable != 0;
    return NEOX_OK;
}

neox_status neox_shard_get_profile(const neox_shard* h, neox_profile* out) {
    if (!h || !out) return NEOX_ERR_INVALID_ARGUMENT;
    *out = h->prof;
    return NEOX_OK;
}

neox_status neox_shard_reset_profile(neox_shard* h) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    const int64_t launches = h->prof.launches;
    h->prof = neox_profile{};
    h->prof.launches = launches;
    return NEOX_OK;
}

neox_status neox_shard_step(neox_shard* h, const void* const* grads, int32_t num_grads, void* params, float lr,
                            void* cuda_stream, neox_step_result* out) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->last_error.clear();
    if (!out) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "out is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    DeviceGuard g(h->device);
    if (!g.ok) return fail(h, NEOX_ERR_CUDA, "cudaSetDevice failed");
    // After asynchronous steps the host copy of t may be behind the device's:
    // then the bias corrections are formed on the device as well.
    if (neox_status s = enqueue_step(h, grads, num_grads, params, lr, nullptr, st, h->async_used, nullptr,
                                     h->profiling);
        s != NEOX_OK)
        return s;
    return read_result(h, st, out);
}

neox_status neox_shard_step_async(neox_shard* h, const void* const* grads, int32_t num_grads, void* params,
                                  float lr, const float* lr_device, void* cuda_stream, neox_step_result* result) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->last_error.clear();
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    DeviceGuard g(h->device);
    if (!g.ok) return fail(h, NEOX_ERR_CUDA, "cudaSetDevice failed");
    h->async_used = true;
    return enqueue_step(h, grads, num_grads, params, lr, lr_device, st, true, result, false);
}

neox_status neox_shard_grad_stats(neox_shard* h, const void* const* grads, int32_t num_grads, void* params,
                                  void* cuda_stream, double* stats_device) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->last_error.clear();
    DeviceGuard g(h->device);
    if (!g.ok) return fail(h, NEOX_ERR_CUDA, "cudaSetDevice failed");
    return enqueue_step(h, grads, num_grads, params, 0.0f, nullptr, static_cast<cudaStream_t>(cuda_stream), false,
                        nullptr, false, kStatsOnly, stats_device);
}

neox_status neox_shard_apply(neox_shard* h, const void* const* grads, int32_t num_grads, void* params, float lr,
                             const double* stats_device, void* cuda_stream, neox_step_result* out) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->last_error.clear();
    if (!out) return fail(h, NEOX_ERR_INVALID_ARGUMENT, "out is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    DeviceGuard g(h->device);
    if (!g.ok) return fail(h, NEOX_ERR_CUDA, "cudaSetDevice failed");
    if (neox_status s = enqueue_step(h, grads, num_grads, params, lr, nullptr, st, h->async_used, nullptr,
                                     h->profiling, kApply, const_cast<double*>(stats_device));
        s != NEOX_OK)
        return s;
    return read_result(h, st, out);
}

}  // extern "C"

// ====================================================================== no-allocation step
//
// neox_shard_step_noalloc runs the same two kernels as neox_shard_step, but
// without a handle and without allocating anything: the per-block partial
// sums, the scalar block and the segment table live in one file-scope static
// device array instead of memory obtained from cudaMalloc at create time.  It
// exists for callers that must not allocate device or pinned memory, e.g. code
// running inside an allocator's own hook (a cudaMalloc there would re-enter
// the allocator), runtimes that hand the whole device memory to their own pool
// up front, and latency-critical loops where cudaMalloc / cudaFree would
// synchronise the device.

#include <mutex>

namespace {

constexpr int kNoallocMaxSegments = 1024;
constexpr int kNoallocMaxParts = 148 * kMaxBlocksPerSm;  // one slot per pass-1 block on a B200
constexpr int kNoallocMaxDevices = 64;

// Byte layout of the static scratch.
constexpr size_t kNaOffScalars = 0;
constexpr size_t kNaOffPartS = 256;
constexpr size_t kNaOffPartB = kNaOffPartS + sizeof(double) * kNoallocMaxParts;
constexpr size_t kNaOffSegEnd = (kNaOffPartB + sizeof(int) * kNoallocMaxParts + 255) / 256 * 256;
constexpr size_t kNaOffSegWd = kNaOffSegEnd + sizeof(unsigned long long) * kNoallocMaxSegments;
constexpr size_t kNoallocScratchBytes = (kNaOffSegWd + sizeof(float) * kNoallocMaxSegments + 255) / 256 * 256;

// Every GPU that loads this library holds these bytes (about 68 KiB) until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct NoallocDevice {
    bool ready = false;
    unsigned long long ctx_id = 0;  // the context the set-up was done in (0: unknown)
    unsigned char* base = nullptr;  // device address of g_noalloc_scratch in that context
    int sm_count = 0;
};
NoallocDevice g_noalloc_dev[kNoallocMaxDevices];
std::mutex g_noalloc_mu;
thread_local char g_noalloc_error[256];

neox_status noalloc_fail(neox_status st, const char* fmt, long long a = 0, long long b = 0) {
    snprintf(g_noalloc_error, sizeof(g_noalloc_error), fmt, a, b);
    return st;
}

// Load one kernel instance onto the current device and cache its occupancy.
// CUDA loads kernels lazily, at their first launch, by default; a load takes
// device memory for the code, so the set-up does it for every instance the
// allocation-free step can launch.  The occupancy cache is filled at the same
// time, so later calls only look it up.
template <class Kern>
cudaError_t noalloc_load(Kern kern, int threads) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, kern);
    if (e == cudaSuccess) (void)occupancy(kern, threads);
    return e;
}

template <class G>
cudaError_t noalloc_load_pass1() {
    cudaError_t e;
    if ((e = noalloc_load(grad_stats_kernel<G, 8, false>, kThreads1)) != cudaSuccess) return e;
    if ((e = noalloc_load(grad_stats_kernel<G, 4, false>, kThreads1)) != cudaSuccess) return e;
    if ((e = noalloc_load(grad_stats_kernel<G, 2, false>, kThreads1)) != cudaSuccess) return e;
    return noalloc_load(grad_stats_kernel<G, 1, false>, kThreads1);
}

// Pass 2 without the FP32 sum and without weight copies (the step has
// neither): AdamW and SGD, chunked and grid-stride.
template <class G, class W, int VEC>
cudaError_t noalloc_load_pass2() {
    cudaError_t e;
    if ((e = noalloc_load(adam_kernel<G, W, VEC, false, false, true>, kThreads3)) != cudaSuccess) return e;
    if ((e = noalloc_load(adam_kernel<G, W, VEC, false, false, false>, kThreads3)) != cudaSuccess) return e;
    if ((e = noalloc_load(sgd_kernel<G, W, VEC, false, false, true>, kThreads3)) != cudaSuccess) return e;
    return noalloc_load(sgd_kernel<G, W, VEC, false, false, false>, kThreads3);
}

template <class G, class W>
cudaError_t noalloc_load_pass2_all() {
    cudaError_t e;
    if ((e = noalloc_load_pass2<G, W, 8>()) != cudaSuccess) return e;
    if ((e = noalloc_load_pass2<G, W, 4>()) != cudaSuccess) return e;
    if ((e = noalloc_load_pass2<G, W, 2>()) != cudaSuccess) return e;
    return noalloc_load_pass2<G, W, 1>();
}

cudaError_t noalloc_load_all() {
    cudaError_t e;
    if ((e = noalloc_load_pass1<F16>()) != cudaSuccess || (e = noalloc_load_pass1<BF16>()) != cudaSuccess ||
        (e = noalloc_load_pass2_all<F16, F16>()) != cudaSuccess ||
        (e = noalloc_load_pass2_all<F16, BF16>()) != cudaSuccess ||
        (e = noalloc_load_pass2_all<BF16, F16>()) != cudaSuccess ||
        (e = noalloc_load_pass2_all<BF16, BF16>()) != cudaSuccess)
        return e;
    return cudaSuccess;
}

// The unique ID of the calling thread's current context (0 if it cannot be
// read).  A context that was destroyed and created again (cudaDeviceReset)
// has a new ID, and the static array and the loaded kernels have to be set
// up again in it.  The two driver functions are taken through the runtime,
// so the library does not link the driver library itself.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {  // under g_noalloc_mu
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// With `dev` current: look up where the static scratch lives on it (host code
// cannot use the array's name as a device address), checking the return
// code, and -- once per device and context -- load every kernel instance the
// step can launch.  The address is looked up on every call (it allocates
// nothing); the rest is redone only when the context changed.
neox_status noalloc_setup(int dev, NoallocDevice** out) {
    if (dev < 0 || dev >= kNoallocMaxDevices) return noalloc_fail(NEOX_ERR_UNSUPPORTED, "device index beyond 63");
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocDevice& d = g_noalloc_dev[dev];
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
        return noalloc_fail(NEOX_ERR_CUDA, "cudaGetSymbolAddress failed (cudaError %lld)", (long long)e);
    const unsigned long long ctx = current_context_id();
    if (!d.ready || ctx != d.ctx_id || p != d.base) {
        d.ready = false;
        int major = 0, sms = 0;
        e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return noalloc_fail(NEOX_ERR_CUDA, "cudaDeviceGetAttribute failed (cudaError %lld)", (long long)e);
        if (major != 10) return noalloc_fail(NEOX_ERR_UNSUPPORTED, "this library is built for sm_100a (B200)");
        if ((e = noalloc_load_all()) != cudaSuccess)
            return noalloc_fail(NEOX_ERR_CUDA, "loading the step's kernels failed (cudaError %lld)", (long long)e);
        d.base = static_cast<unsigned char*>(p);
        d.sm_count = sms;
        d.ctx_id = ctx;
        d.ready = true;
    }
    *out = &d;
    return NEOX_OK;
}

}  // namespace

extern "C" {

const char* neox_noalloc_last_error(void) { return g_noalloc_error; }

neox_status neox_shard_step_noalloc(const neox_shard_desc* d, const neox_hparams* hp, neox_scaler_state* state,
                                    const void* const* grads, int32_t num_grads, void* params, float lr,
                                    void* cuda_stream, neox_step_result* out) {
    g_noalloc_error[0] = 0;
    if (!d || !state || !out) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "desc, state and out must be non-NULL");
    if (const char* why = check_hparams(hp)) {
        snprintf(g_noalloc_error, sizeof(g_noalloc_error), "%s", why);
        return NEOX_ERR_INVALID_ARGUMENT;
    }
    if (hp->hysteresis > 1)
        return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "hysteresis %lld needs a handle (neox_shard_create): the "
                            "scaler state of this call has no hysteresis count", hp->hysteresis);
    if ((d->wdtype != NEOX_FP16 && d->wdtype != NEOX_BF16) || (d->gdtype != NEOX_FP16 && d->gdtype != NEOX_BF16))
        return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "dtype must be NEOX_FP16 or NEOX_BF16");
    if (!(state->scale > 0.0f) || !finite(state->scale) || state->good < 0 || state->t < 0)
        return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "state needs a finite scale > 0, good >= 0, t >= 0");
    if (num_grads < 1 || num_grads > kMaxGrads) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "num_grads must be in [1, 64]");
    if (!grads) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "grads is NULL");
    if (!finite(lr) || lr < 0.0f) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "lr must be finite and >= 0");
    if (!finite(d->default_weight_decay)) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "weight decay must be finite");
    const int nsegs = d->segs ? d->nsegs : 1;
    if (d->segs && nsegs < 1) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "nsegs must be >= 1 with a table");
    if (nsegs > kNoallocMaxSegments)
        return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT,
                            "segment table of %lld entries exceeds the static scratch maximum of %lld segments",
                            nsegs, kNoallocMaxSegments);
    unsigned long long ends[kNoallocMaxSegments];
    float wds[kNoallocMaxSegments];
    if (d->segs) {
        unsigned long long pos = 0;
        for (int i = 0; i < nsegs; i++) {
            const neox_segment& s = d->segs[i];
            if (s.offset != pos || s.numel == 0 || !finite(s.weight_decay))
                return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "segments must be sorted, non-empty, finite and tile [0, numel)");
            pos += s.numel;
            ends[i] = pos;
            wds[i] = s.weight_decay;
        }
        if (pos != d->numel) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "segments do not cover numel");
    } else {
        ends[0] = d->numel;
        wds[0] = d->default_weight_decay;
    }
    GradPtrs gp{};
    uintptr_t a16[kMaxGrads + 1];
    if (d->numel > 0) {
        if (!d->master || !d->exp_avg || !d->exp_avg_sq || !params)
            return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "master/exp_avg/exp_avg_sq/params must be non-NULL");
        if (((uintptr_t)d->master | (uintptr_t)d->exp_avg | (uintptr_t)d->exp_avg_sq) & 3u)
            return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "FP32 state arrays must be 4-byte aligned");
        if ((uintptr_t)params & 1u) return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "params must be 2-byte aligned");
        for (int k = 0; k < num_grads; k++) {
            if (!grads[k] || ((uintptr_t)grads[k] & 1u))
                return noalloc_fail(NEOX_ERR_INVALID_ARGUMENT, "grads[%lld] is NULL or not 2-byte aligned", k);
            gp.p[k] = static_cast<const uint16_t*>(grads[k]);
            a16[k] = (uintptr_t)grads[k];
        }
        a16[num_grads] = (uintptr_t)params;
    }

    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return noalloc_fail(NEOX_ERR_CUDA, "cudaGetDevice failed (cudaError %lld)", (long long)e);
    NoallocDevice* nd = nullptr;
    if (neox_status s = noalloc_setup(dev, &nd); s != NEOX_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);

    // A view of the static scratch shaped like a handle, so the launches below
    // are exactly those of neox_shard_step.  Nothing here allocates.
    neox_shard v;
    v.device = dev;
    v.sm_count = nd->sm_count;
    v.max_parts = nd->sm_count * kMaxBlocksPerSm < kNoallocMaxParts ? nd->sm_count * kMaxBlocksPerSm : kNoallocMaxParts;
    v.numel = d->numel;
    v.hp = *hp;
    v.master = d->master;
    v.m = d->exp_avg;
    v.v = d->exp_avg_sq;
    v.d_sc = reinterpret_cast<DevScalars*>(nd->base + kNaOffScalars);
    v.d_part_s = reinterpret_cast<double*>(nd->base + kNaOffPartS);
    v.d_part_b = reinterpret_cast<int*>(nd->base + kNaOffPartB);
    v.d_seg_end = reinterpret_cast<unsigned long long*>(nd->base + kNaOffSegEnd);
    v.d_seg_wd = reinterpret_cast<float*>(nd->base + kNaOffSegWd);
    v.nsegs = nsegs;

    // The scratch keeps the previous call's contents: reload the scaler block
    // (ticket counter back to zero) and the segment table on this stream.
    DevScalars init{};
    init.scale = state->scale;
    init.scale_used = state->scale;
    init.good = state->good;
    init.t = state->t;
    init.hyst = 1;
    if ((e = cudaMemcpyAsync(v.d_sc, &init, sizeof(init), cudaMemcpyHostToDevice, st)) != cudaSuccess ||
        (e = cudaMemcpyAsync(v.d_seg_end, ends, sizeof(unsigned long long) * nsegs, cudaMemcpyHostToDevice, st)) != cudaSuccess ||
        (e = cudaMemcpyAsync(v.d_seg_wd, wds, sizeof(float) * nsegs, cudaMemcpyHostToDevice, st)) != cudaSuccess)
        return noalloc_fail(NEOX_ERR_CUDA, "staging the scratch failed (cudaError %lld)", (long long)e);

    uintptr_t a32[3] = {(uintptr_t)d->master, (uintptr_t)d->exp_avg, (uintptr_t)d->exp_avg_sq};
    int vec = 1;
    Layout L = d->numel > 0 ? choose_layout(d->numel, a16, num_grads + 1, a32, 3, vec) : Layout{0, 0, 0, 0};

    ScalerArgs sa;
    AdamArgs a;
    make_step_args(*hp, num_grads, lr, state->t, false, sa, a);

    // K >= 5 re-reads the K buffers in pass 2 (no FP32-sum buffer: it would
    // need numel * 4 bytes of scratch).
    e = d->gdtype == NEOX_FP16 ? dispatch1v<F16>(&v, vec, gp, num_grads, L, sa, nullptr, st)
                               : dispatch1v<BF16>(&v, vec, gp, num_grads, L, sa, nullptr, st);
    if (e != cudaSuccess) return noalloc_fail(NEOX_ERR_CUDA, "pass-1 launch failed (cudaError %lld)", (long long)e);
    if (d->numel > 0) {
        uint16_t* w = static_cast<uint16_t*>(params);
        if (d->gdtype == NEOX_FP16) {
            e = d->wdtype == NEOX_FP16 ? dispatch2v<F16, F16>(&v, vec, gp, num_grads, nullptr, L, a, w, st)
                                       : dispatch2v<F16, BF16>(&v, vec, gp, num_grads, nullptr, L, a, w, st);
        } else {
            e = d->wdtype == NEOX_FP16 ? dispatch2v<BF16, F16>(&v, vec, gp, num_grads, nullptr, L, a, w, st)
                                       : dispatch2v<BF16, BF16>(&v, vec, gp, num_grads, nullptr, L, a, w, st);
        }
        if (e != cudaSuccess) return noalloc_fail(NEOX_ERR_CUDA, "pass-2 launch failed (cudaError %lld)", (long long)e);
    }
    DevScalars r{};
    if ((e = cudaMemcpyAsync(&r, v.d_sc, sizeof(r), cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
        return noalloc_fail(NEOX_ERR_CUDA, "step execution failed (cudaError %lld)", (long long)e);
    out->overflow = r.overflow;
    out->grad_norm = r.norm;
    out->clip_coef = r.coef;
    out->loss_scale = r.scale_used;
    out->loss_scale_next = r.scale;
    out->good_steps = r.good;
    out->applied_steps = r.t;
    state->scale = r.scale;
    state->good = r.good;
    state->t = r.t;
    return NEOX_OK;
}

}  // extern "C"
