// neox_multi.cu -- the per-rank mixed-precision optimizer step over a shard
// made of many separately allocated tensors (per-parameter sharding, as in
// FSDP with one shard per parameter), in one pair of launches.
//
// The step is the flat step of neox_shard.cu over the concatenation of the
// tensors, each tensor being one weight-decay segment: the same ingest,
// overflow flag, global norm, loss scaler, clip coefficient, AdamW and cast,
// with the same per-element arithmetic (neox_common.cuh).  Pages followed:
// "OPT: Open Pre-trained Transformer Language Models" (ai-papers.xuzou.cn
// summary), "方法适配" (method adaptation) and "计算设置" (compute setup): FSDP
// shards model state across ranks, Adam state FP32, weights FP16, dynamic
// loss scaling, gradient pre-divide and clipping.
//
// Work decomposition.  Each tensor keeps its own vector width and peeled
// head, chosen from its own pointers; its head and ragged tail are done by
// block (tensor index mod grid).  The tensors whose arrays share a 16-byte
// residue -- nearly always all of them -- stream 8-element vectors, and their
// vectors form one sequence, tensor after tensor (the MtSeq table):
//  * Pass 1 deals the sequence to the threads with a fixed assignment
//    (thread g takes vectors g, g + S, g + 2S, ...; S = threads of the grid),
//    four per batch, so the norm is deterministic and the batches run full
//    across tensor ends.  On the Pythia-1.4B layout as 290 tensors the
//    earlier per-tensor grid-stride, whose last batch of every tensor ran
//    partly empty and which formed each tensor's starting thread with a
//    64-bit modulo, took 0.59 ms against 0.44 for the flat pass.
//  * The SGD pass takes the sequence in chunks of four-vector batches from
//    the counter in the scalar block, as the flat SGD pass does.
//  * The AdamW pass takes the vectors of all tensors (any width) as one
//    sequence in chunks from the same counter, as the flat AdamW pass does.
// Tensors with narrower vectors are covered grid-stride, tensor by tensor,
// after the sequence.  A static decomposition into per-block chunks (every
// block streaming its own distant region) was measured 11% slower than the
// grid-stride.

#include "neox_shard.h"
#include "neox_common.cuh"

#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

namespace {

constexpr int kMtThreads1 = 512;
constexpr int kMtThreads3 = 256;
constexpr int kMtChunk = 2;        // pass 2 (AdamW): vectors per thread in each chunk taken from the counter

struct alignas(16) MtTensor {
    float* master;
    float* m;
    float* v;
    uint16_t* w;
    unsigned long long numel, head, nvec;  // the vectors are [head, head + nvec * vec)
    float wd;
    int vec;
    int gbase;  // the tensor's K gradient pointers are gtab[gbase .. gbase + K)
    int pad_;
    // The vectors of all earlier tensors.  A pass's grid-stride starts this
    // tensor where the previous one left off (this count modulo the pass's
    // thread count), so the tensors' vectors are dealt to the threads as one
    // sequence: no thread takes the remainder of every tensor.
    unsigned long long before;
};

static_assert(sizeof(MtTensor) % 16 == 0, "descriptors are copied as 16-byte words");

// This thread's first vector of a tensor that follows `before` vectors of
// earlier tensors (THREADS x gridDim.x threads in all).
template <int THREADS>
__device__ __forceinline__ unsigned long long rotated_start(unsigned long long before) {
    const unsigned long long n = (unsigned long long)gridDim.x * THREADS;
    const unsigned long long g = (unsigned long long)blockIdx.x * THREADS + threadIdx.x;
    const unsigned long long r = before % n;
    return g >= r ? g - r : g + n - r;
}

// ---------------------------------------------------------------- pass 1
// The 8-element vectors of all tensors whose layout has VEC = 8 (every tensor
// whose arrays share a 16-byte residue, i.e. nearly always) form one
// sequence, tensor after tensor.  Entry t of this table describes the t-th
// such tensor: sequence vector gv (end_{t-1} <= gv < end_t) is its elements
// off0 + 8 gv ... off0 + 8 gv + 7.
struct alignas(16) MtSeq {
    unsigned long long end;  // one past the tensor's last vector in the sequence
    long long off0;          // element index of sequence vector gv: off0 + 8 * gv
    const uint16_t* g0;      // the tensor's first gradient buffer
    int gbase;               // its K gradient pointers are gtab[gbase .. gbase + K)
    float wd;                // its weight decay
    float* master;           // (the SGD pass) its FP32 master weights
    uint16_t* w;             //                its 16-bit working weights
};
static_assert(sizeof(MtSeq) == 48, "three 16-byte words; pass 1 reads the first two");

// A thread's position in the sequence table.  Its vectors come in increasing
// order, so the cursor only moves forward; over the whole pass a thread
// crosses each tensor boundary at most once.
struct SeqCursor {
    int t = -1;
    unsigned long long end = 0;
    long long off0 = 0;
    const uint16_t* g0 = nullptr;
    int gbase = 0;
    __device__ __forceinline__ void to(const MtSeq* __restrict__ seq, unsigned long long gv) {
        while (gv >= end) {
            ++t;
            const int4 a = __ldg(reinterpret_cast<const int4*>(seq + t));
            const int4 b = __ldg(reinterpret_cast<const int4*>(seq + t) + 1);
            end = (unsigned long long)(unsigned)a.x | ((unsigned long long)(unsigned)a.y << 32);
            off0 = (long long)((unsigned long long)(unsigned)a.z | ((unsigned long long)(unsigned)a.w << 32));
            g0 = reinterpret_cast<const uint16_t*>((unsigned long long)(unsigned)b.x |
                                                   ((unsigned long long)(unsigned)b.y << 32));
            gbase = b.z;
        }
    }
};

// U vectors whose gradient addresses are known, ingested together: for every
// buffer the U loads are issued before any is used.  ok[u] = false leaves
// vector u zero (no load).  Per element the arithmetic is ingest()'s.
template <class G, int U, bool PRED>
__device__ __forceinline__ void seq_ingest(const uint16_t* const (&a0)[U], const long long (&el)[U],
                                           const int (&gb)[U], const bool (&ok)[U],
                                           const uint16_t* const* __restrict__ gtab, int K, float inv_pre,
                                           float inv_us, float (&g)[U][8]) {
    const bool pre1 = inv_pre == 1.0f;  // x * 1 == x exactly: skip the multiply
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < 8; e++) g[u][e] = 0.0f;
    for (int k = 0; k < K; k++) {
        uint16_t h[U][8];
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (!PRED || ok[u]) {
                ld16<8>(k == 0 ? a0[u] : gtab[gb[u] + k] + el[u], h[u]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; e++) h[u][e] = 0;
            }
        }
        if (pre1) {
#pragma unroll
            for (int u = 0; u < U; u++)
#pragma unroll
                for (int e = 0; e < 8; e++) g[u][e] = __fadd_rn(g[u][e], G::dec(h[u][e]));
        } else {
#pragma unroll
            for (int u = 0; u < U; u++)
#pragma unroll
                for (int e = 0; e < 8; e++) g[u][e] = __fadd_rn(g[u][e], __fmul_rn(G::dec(h[u][e]), inv_pre));
        }
    }
#pragma unroll
    for (int u = 0; u < U; u++)
#pragma unroll
        for (int e = 0; e < 8; e++) g[u][e] = __fmul_rn(g[u][e], inv_us);
}

// Pass 1 over the sequence, with a fixed assignment of vectors to threads:
// thread g takes sequence vectors g, g + S, g + 2S, ... (S = threads of the
// grid), U of them per batch whose loads are issued together, and sums its
// squares in that order, so the norm is deterministic.  The batches run full
// across tensor ends (a per-tensor grid-stride leaves the last batch of every
// tensor partly empty).  A batch whose U vectors lie in one tensor -- nearly
// every batch, the vectors being S apart -- addresses them from one base as
// the flat pass does; a batch across a tensor end moves the cursor vector by
// vector; the last, partial batch is predicated.
template <class G, int KFIX>
__device__ __forceinline__ void mt_p1_seq(const MtSeq* __restrict__ seq, unsigned long long total,
                                          const uint16_t* const* __restrict__ gtab, int K_rt, float inv_pre,
                                          float inv_us, double& s, int& bad) {
    const int K = KFIX ? KFIX : K_rt;
    constexpr int U = KFIX ? 4 : 2;
    const unsigned long long S = (unsigned long long)gridDim.x * kMtThreads1;
    SeqCursor cur;
    unsigned long long v = (unsigned long long)blockIdx.x * kMtThreads1 + threadIdx.x;
    for (; v + (U - 1) * S < total; v += U * S) {
        cur.to(seq, v);
        const uint16_t* a0[U];
        long long el[U];
        int gb[U];
        const bool ok[U] = {};
        float g[U][8];
        if (v + (U - 1) * S < cur.end) {  // one tensor: one base, constant strides
#pragma unroll
            for (int u = 0; u < U; u++) {
                el[u] = cur.off0 + 8ll * (long long)v + 8ll * (long long)(u * S);
                a0[u] = cur.g0 + el[u];
                gb[u] = cur.gbase;
            }
        } else {
#pragma unroll
            for (int u = 0; u < U; u++) {
                cur.to(seq, v + u * S);
                el[u] = cur.off0 + 8ll * (long long)(v + u * S);
                a0[u] = cur.g0 + el[u];
                gb[u] = cur.gbase;
            }
        }
        seq_ingest<G, U, false>(a0, el, gb, ok, gtab, K, inv_pre, inv_us, g);
#pragma unroll
        for (int u = 0; u < U; u++) s += vec_sumsq<8>(g[u], bad);
    }
    if (v < total) {  // the last, partial batch
        const uint16_t* a0[U];
        long long el[U];
        int gb[U];
        bool ok[U];
        float g[U][8];
#pragma unroll
        for (int u = 0; u < U; u++) {
            ok[u] = v + u * S < total;
            if (ok[u]) cur.to(seq, v + u * S);
            el[u] = cur.off0 + 8ll * (long long)(v + u * S);
            a0[u] = cur.g0 + el[u];
            gb[u] = cur.gbase;
        }
        seq_ingest<G, U, true>(a0, el, gb, ok, gtab, K, inv_pre, inv_us, g);
#pragma unroll
        for (int u = 0; u < U; u++)
            if (ok[u]) s += vec_sumsq<8>(g[u], bad);
    }
}

// Pass 1 over one tensor with narrower vectors (arrays without a common
// 16-byte residue), grid-stride across the whole grid from the tensor's
// rotated start, U strides per batch.
template <class G, int VEC, int KFIX>
__device__ __forceinline__ void mt_p1_tensor(const GradTab& gp, int K_rt, const MtTensor& T, float inv_pre,
                                             float inv_us, double& s, int& bad) {
    const int K = KFIX ? KFIX : K_rt;
    constexpr int U = KFIX ? 4 : 2;
    const unsigned long long stride = (unsigned long long)gridDim.x * kMtThreads1;
    unsigned long long v = rotated_start<kMtThreads1>(T.before);
    for (; v + (U - 1) * stride < T.nvec; v += U * stride) {
        float g[U][VEC];
        ingest_batch<G, VEC, U>(gp, K, T.head + v * VEC, stride * VEC, inv_pre, inv_us, g);
#pragma unroll
        for (int u = 0; u < U; u++) s += vec_sumsq<VEC>(g[u], bad);
    }
    if (v < T.nvec) {
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; u++) ok[u] = v + u * stride < T.nvec;
        float g[U][VEC];
        ingest_batch_pred<G, VEC, U>(gp, K, T.head + v * VEC, stride * VEC, ok, inv_pre, inv_us, g);
#pragma unroll
        for (int u = 0; u < U; u++)
            if (ok[u]) s += vec_sumsq<VEC>(g[u], bad);
    }
}

template <class G, int KFIX>
__device__ __forceinline__ void mt_p1_dispatch(const MtTensor& T, const GradTab& gp, int K, float inv_pre,
                                               float inv_us, double& s, int& bad) {
    switch (T.vec) {
        case 4: mt_p1_tensor<G, 4, KFIX>(gp, K, T, inv_pre, inv_us, s, bad); break;
        case 2: mt_p1_tensor<G, 2, KFIX>(gp, K, T, inv_pre, inv_us, s, bad); break;
        default: mt_p1_tensor<G, 1, KFIX>(gp, K, T, inv_pre, inv_us, s, bad); break;
    }
}

// Pass 1: the sequence of 8-element vectors, then the tensors with narrower
// vectors (`odd`, normally none), then every tensor's peeled head and ragged
// tail (tensor t by block t mod grid), each thread summing in that fixed
// order; then the shared end of pass 1 (finish_pass1).
template <class G>
__global__ void __launch_bounds__(kMtThreads1, 1024 / kMtThreads1)
mt_stats_kernel(const MtTensor* __restrict__ tens, int ntensors, const MtSeq* __restrict__ seq,
                unsigned long long total8, const int* __restrict__ odd, int nodd,
                const uint16_t* const* __restrict__ gtab, int K, ScalerArgs sa, double* __restrict__ part_s,
                int* __restrict__ part_b, DevScalars* __restrict__ sc) {
    __shared__ double sh_s[kMtThreads1 / 32];
    __shared__ int sh_b[kMtThreads1 / 32];
    __shared__ bool is_last;
    const float inv_us = unscale_factor(sa.post, sc->scale);
    double s = 0.0;
    int bad = 0;
    if (K == 1) mt_p1_seq<G, 1>(seq, total8, gtab, K, sa.inv_pre, inv_us, s, bad);
    else mt_p1_seq<G, 0>(seq, total8, gtab, K, sa.inv_pre, inv_us, s, bad);
    for (int j = 0; j < nodd; j++) {
        const MtTensor T = tens[__ldg(odd + j)];
        const GradTab gp{gtab, T.gbase};
        if (K == 1) mt_p1_dispatch<G, 1>(T, gp, K, sa.inv_pre, inv_us, s, bad);
        else mt_p1_dispatch<G, 0>(T, gp, K, sa.inv_pre, inv_us, s, bad);
    }
    for (int ti = blockIdx.x; ti < ntensors; ti += gridDim.x) {  // heads and ragged tails
        const MtTensor T = tens[ti];
        if (T.numel == 0) continue;
        const GradTab gp{gtab, T.gbase};
        const unsigned long long tail0 = T.head + T.nvec * T.vec;
        const unsigned long long extra = T.head + (T.numel - tail0);
        for (unsigned long long j = threadIdx.x; j < extra; j += kMtThreads1) {
            const unsigned long long i = j < T.head ? j : tail0 + (j - T.head);
            float g[1];
            ingest<G, 1>(gp, K, i, sa.inv_pre, inv_us, g);
            s += vec_sumsq<1>(g, bad);
        }
    }
    finish_pass1<kMtThreads1>(s, bad, part_s, part_b, sc, sa, sh_s, sh_b, &is_last);
}

// ---------------------------------------------------------------- pass 2
// Pass 2 with plain SGD over one tensor with narrower vectors, grid-stride
// from the tensor's rotated start, kUnrollSgd strides in flight per thread
// (its loads are too few per vector to cover the memory latency one at a
// time).
template <class G, class W, int VEC, int KFIX>
__device__ __forceinline__ void mt_sgd_tensor(const GradTab& gp, int K_rt, const MtTensor& T, float keep1, float c,
                                              float inv_us, const AdamArgs& a) {
    const int K = KFIX ? KFIX : K_rt;
    float keep[VEC];
#pragma unroll
    for (int e = 0; e < VEC; e++) keep[e] = keep1;
    const unsigned long long stride = (unsigned long long)gridDim.x * kMtThreads3;
    float* __restrict__ master = T.master;
    uint16_t* __restrict__ w = T.w;
    const unsigned long long nvec = T.nvec, head = T.head;
    unsigned long long vi = rotated_start<kMtThreads3>(T.before);
    constexpr int U = kUnrollSgd;
    for (; vi + (U - 1) * stride < nvec; vi += U * stride) {
        float g[U][VEC], p[U][VEC];
        ingest_batch<G, VEC, U>(gp, K, head + vi * VEC, stride * VEC, a.inv_pre, inv_us, g);
#pragma unroll
        for (int u = 0; u < U; u++) ld32<VEC>(master + head + (vi + u * stride) * VEC, p[u]);
#pragma unroll
        for (int u = 0; u < U; u++) {
            const unsigned long long i = head + (vi + u * stride) * VEC;
            sgd_vec<VEC>(g[u], keep, c, a.lr, p[u]);
            st32<VEC>(master + i, p[u]);
            st16<W, VEC>(w + i, p[u]);
        }
    }
    for (; vi < nvec; vi += stride) {
        const unsigned long long i = head + vi * VEC;
        float g[VEC], p[VEC];
        ingest<G, VEC>(gp, K, i, a.inv_pre, inv_us, g);
        ld32<VEC>(master + i, p);
        sgd_vec<VEC>(g, keep, c, a.lr, p);
        st32<VEC>(master + i, p);
        st16<W, VEC>(w + i, p);
    }
}

template <class G, class W, int KFIX>
__device__ __forceinline__ void mt_sgd_dispatch(const MtTensor& T, const GradTab& gp, int K, float keep1, float c,
                                                float inv_us, const AdamArgs& a) {
    switch (T.vec) {
        case 4: mt_sgd_tensor<G, W, 4, KFIX>(gp, K, T, keep1, c, inv_us, a); break;
        case 2: mt_sgd_tensor<G, W, 2, KFIX>(gp, K, T, keep1, c, inv_us, a); break;
        default: mt_sgd_tensor<G, W, 1, KFIX>(gp, K, T, keep1, c, inv_us, a); break;
    }
}

// The sequence cursor of the SGD pass: pass 1's, plus the tensor's master
// and working-weight arrays and its decay factor fl32(1 - fl32(lr * wd)).
struct SeqCursor2 {
    int t = -1;
    unsigned long long start = 0;  // the tensor's first vector in the sequence
    unsigned long long end = 0;
    long long off0 = 0;
    const uint16_t* g0 = nullptr;
    int gbase = 0;
    float keep = 1.0f;
    float* master = nullptr;
    uint16_t* w = nullptr;
    __device__ __forceinline__ void to(const MtSeq* __restrict__ seq, unsigned long long gv, float lr) {
        while (gv >= end) {
            ++t;
            const int4* q = reinterpret_cast<const int4*>(seq + t);
            const int4 a = __ldg(q), b = __ldg(q + 1), d = __ldg(q + 2);
            start = end;
            end = (unsigned long long)(unsigned)a.x | ((unsigned long long)(unsigned)a.y << 32);
            off0 = (long long)((unsigned long long)(unsigned)a.z | ((unsigned long long)(unsigned)a.w << 32));
            g0 = reinterpret_cast<const uint16_t*>((unsigned long long)(unsigned)b.x |
                                                   ((unsigned long long)(unsigned)b.y << 32));
            gbase = b.z;
            keep = __fsub_rn(1.0f, __fmul_rn(lr, __int_as_float(b.w)));
            master = reinterpret_cast<float*>((unsigned long long)(unsigned)d.x | ((unsigned long long)(unsigned)d.y << 32));
            w = reinterpret_cast<uint16_t*>((unsigned long long)(unsigned)d.z | ((unsigned long long)(unsigned)d.w << 32));
        }
    }
};

// Pass 2 with plain SGD: the sequence of 8-element vectors in chunks of
// kUnrollSgd x kMtThreads3 vectors taken from the counter in the scalar block
// (zeroed by pass 1's last block, which this grid waits for) -- the flat SGD
// pass's scheme.  When a warp's kUnrollSgd tiles lie in one tensor, as in
// nearly every chunk, they take the split tiles of the flat passes, loaded as
// one batch; otherwise a thread's vectors are loaded as one batch when they
// lie in one tensor, and one at a time across a tensor end.  The cursor only
// moves forward: a block's chunks, and a thread's vectors in a chunk, come in
// increasing order.
template <class G, class W>
__device__ __forceinline__ void mt_sgd_seq(const MtSeq* __restrict__ seq, unsigned long long total,
                                           const uint16_t* const* __restrict__ gtab, int K, float c, float inv_us,
                                           const AdamArgs& a, DevScalars* __restrict__ sc) {
    constexpr int U = kUnrollSgd;
    constexpr unsigned long long kChunk = (unsigned long long)kMtThreads3 * U;
    constexpr unsigned long long kDi = (unsigned long long)kMtThreads3 * 8;  // elements between a thread's vectors
    const unsigned long long nchunks = (total + kChunk - 1) / kChunk;
    __shared__ unsigned int chunk_sh;
    SeqCursor2 cur;
    for (;;) {
        if (threadIdx.x == 0) chunk_sh = atomicAdd(&sc->chunk_next, 1u);
        __syncthreads();
        const unsigned long long ch = chunk_sh;
        __syncthreads();                  // chunk_sh is rewritten by the next iteration
        if (ch >= nchunks) break;         // uniform across the block
        const unsigned long long gv0 = ch * kChunk + threadIdx.x;
        if (gv0 >= total) continue;
        cur.to(seq, gv0, a.lr);
        const unsigned int lane = threadIdx.x & 31;
        const unsigned long long tile = gv0 - lane;  // the warp's 32 consecutive vectors start here
        if (tile >= cur.start && tile + (U - 1) * kMtThreads3 + 31 < cur.end) {
            // the warp's U tiles lie in one tensor (then every lane of the warp
            // sees it): split them as the flat passes do, lane t taking elements
            // 4t + [0, 4) and 128 + 4t + [0, 4) of each tile, all 2U gradient
            // halves loaded as one batch
            const unsigned long long b0 = (unsigned long long)(cur.off0 + 8ll * (long long)tile) + 4ull * lane;
            const GradTab gp{gtab, cur.gbase};
            float g[U][8], p[U][8], keep[8];
            ingest_halves<G, U>(gp, K, b0, kDi, a.inv_pre, inv_us, g);
#pragma unroll
            for (int u = 0; u < U; u++) {
                float lo[4], hi[4];
                ld32<4>(cur.master + b0 + u * kDi, lo);
                ld32<4>(cur.master + b0 + u * kDi + 128, hi);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    p[u][e] = lo[e];
                    p[u][4 + e] = hi[e];
                }
            }
#pragma unroll
            for (int e = 0; e < 8; e++) keep[e] = cur.keep;
#pragma unroll
            for (int u = 0; u < U; u++) {
                sgd_vec<8>(g[u], keep, c, a.lr, p[u]);
                float lo[4], hi[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    lo[e] = p[u][e];
                    hi[e] = p[u][4 + e];
                }
                st32<4>(cur.master + b0 + u * kDi, lo);
                st32<4>(cur.master + b0 + u * kDi + 128, hi);
                st16<W, 4>(cur.w + b0 + u * kDi, lo);
                st16<W, 4>(cur.w + b0 + u * kDi + 128, hi);
            }
        } else if (gv0 + (U - 1) * kMtThreads3 < cur.end) {  // the thread's U vectors lie in one tensor
            const unsigned long long el0 = (unsigned long long)(cur.off0 + 8ll * (long long)gv0);
            const GradTab gp{gtab, cur.gbase};
            float g[U][8], p[U][8], keep[8];
            ingest_batch<G, 8, U>(gp, K, el0, kDi, a.inv_pre, inv_us, g);
#pragma unroll
            for (int u = 0; u < U; u++) ld32<8>(cur.master + el0 + u * kDi, p[u]);
#pragma unroll
            for (int e = 0; e < 8; e++) keep[e] = cur.keep;
#pragma unroll
            for (int u = 0; u < U; u++) {
                sgd_vec<8>(g[u], keep, c, a.lr, p[u]);
                st32<8>(cur.master + el0 + u * kDi, p[u]);
                st16<W, 8>(cur.w + el0 + u * kDi, p[u]);
            }
        } else {
            for (int u = 0; u < U; u++) {
                const unsigned long long gv = gv0 + (unsigned long long)u * kMtThreads3;
                if (gv >= total) break;
                cur.to(seq, gv, a.lr);
                const unsigned long long el = (unsigned long long)(cur.off0 + 8ll * (long long)gv);
                const GradTab gp{gtab, cur.gbase};
                float g[8], p[8], keep[8];
                ingest<G, 8>(gp, K, el, a.inv_pre, inv_us, g);
                ld32<8>(cur.master + el, p);
#pragma unroll
                for (int e = 0; e < 8; e++) keep[e] = cur.keep;
                sgd_vec<8>(g, keep, c, a.lr, p);
                st32<8>(cur.master + el, p);
                st16<W, 8>(cur.w + el, p);
            }
        }
    }
}

template <class G, class W>
__global__ void __launch_bounds__(kMtThreads3, 2)
mt_sgd_kernel(const MtTensor* __restrict__ tens, int ntensors, const MtSeq* __restrict__ seq,
              unsigned long long total8, const int* __restrict__ odd, int nodd,
              const uint16_t* const* __restrict__ gtab, int K, AdamArgs a_arg, DevScalars* __restrict__ sc) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // pass 1's results
    if (sc->overflow) return;
    const float c = sc->coef;
    AdamArgs a = a_arg;
    const float inv_us = unscale_factor(a.post, sc->scale_used);
    if (a.device_bc) {
        a.lr = sc->lr;
        a.step_size = sc->step_size;
        a.bcs = sc->bc2_sqrt;
    }
    mt_sgd_seq<G, W>(seq, total8, gtab, K, c, inv_us, a, sc);
    for (int j = 0; j < nodd; j++) {
        const MtTensor T = tens[__ldg(odd + j)];
        const GradTab gp{gtab, T.gbase};
        const float keep1 = __fsub_rn(1.0f, __fmul_rn(a.lr, T.wd));  // fl32(1 - fl32(lr * wd))
        if (K == 1) mt_sgd_dispatch<G, W, 1>(T, gp, K, keep1, c, inv_us, a);
        else mt_sgd_dispatch<G, W, 0>(T, gp, K, keep1, c, inv_us, a);
    }
    for (int ti = blockIdx.x; ti < ntensors; ti += gridDim.x) {  // heads and ragged tails
        const MtTensor T = tens[ti];
        if (T.numel == 0) continue;
        const GradTab gp{gtab, T.gbase};
        const float keep1 = __fsub_rn(1.0f, __fmul_rn(a.lr, T.wd));
        const unsigned long long tail0 = T.head + T.nvec * T.vec;
        const unsigned long long extra = T.head + (T.numel - tail0);
        for (unsigned long long j = threadIdx.x; j < extra; j += kMtThreads3) {
            const unsigned long long i = j < T.head ? j : tail0 + (j - T.head);
            float g[1], p[1] = {T.master[i]}, keep[1] = {keep1};
            ingest<G, 1>(gp, K, i, a.inv_pre, inv_us, g);
            sgd_vec<1>(g, keep, c, a.lr, p);
            T.master[i] = p[0];
            T.w[i] = W::enc(p[0]);
        }
    }
}

// One AdamW vector: local vector vi of tensor T.
template <class G, class W, int VEC, int KFIX>
__device__ __forceinline__ void mt_adam_one(const GradTab& gp, int K_rt, const MtTensor& T, unsigned long long vi,
                                            float keep1, float c, float inv_us, const AdamArgs& a) {
    const int K = KFIX ? KFIX : K_rt;
    float keep[VEC];
#pragma unroll
    for (int e = 0; e < VEC; e++) keep[e] = keep1;
    const unsigned long long i = T.head + vi * VEC;
    float g[VEC], p[VEC], mm[VEC], vv[VEC];
    ingest<G, VEC>(gp, K, i, a.inv_pre, inv_us, g);
    ld32<VEC>(T.master + i, p);
    ld32<VEC>(T.m + i, mm);
    ld32<VEC>(T.v + i, vv);
    adam_vec<VEC>(g, keep, c, a, p, mm, vv);
    st32<VEC>(T.master + i, p);
    st32<VEC>(T.m + i, mm);
    st32<VEC>(T.v + i, vv);
    st16<W, VEC>(T.w + i, p);
}

// One AdamW vector of a split tile: elements i0 + [0, 4) and i0 + 128 + [0, 4)
// of tensor T (lane t of a tile whose 32 vectors lie in T takes i0 = the
// tile's first element + 4t), so that each warp-wide FP32 access covers 512
// contiguous bytes.
template <class G, class W, int KFIX>
__device__ __forceinline__ void mt_adam_split(const GradTab& gp, int K_rt, const MtTensor& T, unsigned long long i0,
                                              float keep1, float c, float inv_us, const AdamArgs& a) {
    const int K = KFIX ? KFIX : K_rt;
    const unsigned long long i1 = i0 + 128;
    float g0[4], g1[4], p0[4], p1[4], m0[4], m1[4], v0[4], v1[4], keep[4];
#pragma unroll
    for (int e = 0; e < 4; e++) keep[e] = keep1;
    ingest<G, 4>(gp, K, i0, a.inv_pre, inv_us, g0);
    ingest<G, 4>(gp, K, i1, a.inv_pre, inv_us, g1);
    ld32<4>(T.master + i0, p0);
    ld32<4>(T.master + i1, p1);
    ld32<4>(T.m + i0, m0);
    ld32<4>(T.m + i1, m1);
    ld32<4>(T.v + i0, v0);
    ld32<4>(T.v + i1, v1);
    adam_vec<4>(g0, keep, c, a, p0, m0, v0);
    adam_vec<4>(g1, keep, c, a, p1, m1, v1);
    st32<4>(T.master + i0, p0);
    st32<4>(T.master + i1, p1);
    st32<4>(T.m + i0, m0);
    st32<4>(T.m + i1, m1);
    st32<4>(T.v + i0, v0);
    st32<4>(T.v + i1, v1);
    st16<W, 4>(T.w + i0, p0);
    st16<W, 4>(T.w + i1, p1);
}

template <class G, class W, int KFIX>
__device__ __forceinline__ void mt_adam_one_dispatch(const GradTab& gp, int K, const MtTensor& T,
                                                     unsigned long long vi, float keep1, float c, float inv_us,
                                                     const AdamArgs& a) {
    switch (T.vec) {
        case 8: mt_adam_one<G, W, 8, KFIX>(gp, K, T, vi, keep1, c, inv_us, a); break;
        case 4: mt_adam_one<G, W, 4, KFIX>(gp, K, T, vi, keep1, c, inv_us, a); break;
        case 2: mt_adam_one<G, W, 2, KFIX>(gp, K, T, vi, keep1, c, inv_us, a); break;
        default: mt_adam_one<G, W, 1, KFIX>(gp, K, T, vi, keep1, c, inv_us, a); break;
    }
}

// Pass 2 with AdamW: the vectors of all tensors form one sequence (tensor t
// holds [before_t, before_t + nvec_t)), handed out in chunks of kMtChunk x
// kMtThreads3 vectors from the counter in the scalar block (zeroed by pass
// 1's last block, which this grid waits for), so that SMs served faster take
// more, as in the flat pass.  Each thread keeps a tensor cursor, which only
// moves forward because a block's chunks come in increasing order.  Heads and
// tails: tensor t's by block (t mod grid).  Held to 64 registers for 4 blocks
// per SM (a few spilled descriptor fields are read only at tensor changes):
// on the Pythia-1.4B layout as 290 tensors this measured 211 Gparams/s,
// against 199 at 3 blocks per SM and 205 for the per-tensor grid-stride.
template <class G, class W>
__global__ void __launch_bounds__(kMtThreads3, 4)
mt_adam_chunked_kernel(const MtTensor* __restrict__ tens, int ntensors, const uint16_t* const* __restrict__ gtab,
                       int K, AdamArgs a_arg, DevScalars* __restrict__ sc, unsigned long long total_vecs) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // pass 1's results
    if (sc->overflow) return;
    const float c = sc->coef;
    AdamArgs a = a_arg;
    const float inv_us = unscale_factor(a.post, sc->scale_used);
    if (a.device_bc) {
        a.lr = sc->lr;
        a.step_size = sc->step_size;
        a.bcs = sc->bc2_sqrt;
    }
    constexpr unsigned long long kChunk = (unsigned long long)kMtThreads3 * kMtChunk;
    const unsigned long long nchunks = (total_vecs + kChunk - 1) / kChunk;
    __shared__ unsigned int chunk_sh;
    int t = -1;
    MtTensor T{};
    unsigned long long tend = 0;  // one past tensor t's last vector in the sequence
    float keep1 = 1.0f;
    for (;;) {
        if (threadIdx.x == 0) chunk_sh = atomicAdd(&sc->chunk_next, 1u);
        __syncthreads();
        const unsigned long long ch = chunk_sh;
        __syncthreads();                  // chunk_sh is rewritten by the next iteration
        if (ch >= nchunks) break;         // uniform across the block
        for (int k = 0; k < kMtChunk; k++) {
            const unsigned long long gv = ch * kChunk + (unsigned long long)k * kMtThreads3 + threadIdx.x;
            if (gv >= total_vecs) break;
            while (gv >= tend) {          // gv < total_vecs = the last tensor's end: t stays < ntensors
                ++t;
                T = tens[t];
                tend = T.before + T.nvec;
                keep1 = __fsub_rn(1.0f, __fmul_rn(a.lr, T.wd));  // fl32(1 - fl32(lr * wd))
            }
            const GradTab gp{gtab, T.gbase};
            const unsigned int lane = threadIdx.x & 31;
            const unsigned long long tile = gv - lane;  // the warp's 32 consecutive vectors
            if (T.vec == 8 && tile >= T.before && tile + 31 < tend) {
                // the tile lies in T (so every lane of the warp sees it): split it
                const unsigned long long i0 = T.head + 8 * (tile - T.before) + 4ull * lane;
                if (K == 1) mt_adam_split<G, W, 1>(gp, K, T, i0, keep1, c, inv_us, a);
                else mt_adam_split<G, W, 0>(gp, K, T, i0, keep1, c, inv_us, a);
            } else if (K == 1) {
                mt_adam_one_dispatch<G, W, 1>(gp, K, T, gv - T.before, keep1, c, inv_us, a);
            } else {
                mt_adam_one_dispatch<G, W, 0>(gp, K, T, gv - T.before, keep1, c, inv_us, a);
            }
        }
    }
    for (int ti = blockIdx.x; ti < ntensors; ti += gridDim.x) {  // heads and tails
        const MtTensor H = tens[ti];
        if (H.numel == 0) continue;
        const GradTab gp{gtab, H.gbase};
        const float kh = __fsub_rn(1.0f, __fmul_rn(a.lr, H.wd));
        const unsigned long long tail0 = H.head + H.nvec * H.vec;
        const unsigned long long extra = H.head + (H.numel - tail0);
        for (unsigned long long j = threadIdx.x; j < extra; j += kMtThreads3) {
            const unsigned long long i = j < H.head ? j : tail0 + (j - H.head);
            float g[1], p[1] = {H.master[i]}, mm[1] = {H.m[i]}, vv[1] = {H.v[i]}, keep[1] = {kh};
            ingest<G, 1>(gp, K, i, a.inv_pre, inv_us, g);
            adam_vec<1>(g, keep, c, a, p, mm, vv);
            H.master[i] = p[0];
            H.m[i] = mm[0];
            H.v[i] = vv[0];
            H.w[i] = W::enc(p[0]);
        }
    }
}

using MtSgdKernel = void (*)(const MtTensor*, int, const MtSeq*, unsigned long long, const int*, int,
                             const uint16_t* const*, int, AdamArgs, DevScalars*);
using MtAdamKernel = void (*)(const MtTensor*, int, const uint16_t* const*, int, AdamArgs, DevScalars*,
                              unsigned long long);

MtSgdKernel mt_sgd_kernel_for(neox_dtype gdt, neox_dtype wdt) {
    return gdt == NEOX_FP16 ? (wdt == NEOX_FP16 ? mt_sgd_kernel<F16, F16> : mt_sgd_kernel<F16, BF16>)
                            : (wdt == NEOX_FP16 ? mt_sgd_kernel<BF16, F16> : mt_sgd_kernel<BF16, BF16>);
}

MtAdamKernel mt_adam_kernel_for(neox_dtype gdt, neox_dtype wdt) {
    return gdt == NEOX_FP16 ? (wdt == NEOX_FP16 ? mt_adam_chunked_kernel<F16, F16> : mt_adam_chunked_kernel<F16, BF16>)
                            : (wdt == NEOX_FP16 ? mt_adam_chunked_kernel<BF16, F16> : mt_adam_chunked_kernel<BF16, BF16>);
}

}  // namespace

// ====================================================================== host

struct neox_multi {
    int device = 0;
    int sm_count = 0;
    int ntensors = 0;
    int K = 1;
    neox_dtype wdtype = NEOX_FP16, gdtype = NEOX_FP16;
    neox_hparams hp{};
    unsigned long long numel = 0;
    unsigned long long total_vecs = 0;  // vectors of all tensors
    int grid1 = 1;                      // pass-1 grid (set at create)
    int grid2 = 1, grid2_sgd = 1;       // pass-2 grids of the two update rules (set at create)
    float scale = 1.0f;
    int32_t good = 0;
    long long t = 0;
    bool async_used = false;
    int max_parts = 0;
    MtTensor* d_tens = nullptr;
    const uint16_t** d_gtab = nullptr;
    MtSeq* d_seq = nullptr;             // pass 1: the sequence of 8-element vectors
    int* d_odd = nullptr;               // pass 1: tensors with narrower vectors
    int nseq = 0, nodd = 0;
    unsigned long long total8 = 0;      // vectors in the sequence
    std::vector<int> seq_tensor;        // tensor index of each sequence entry
    DevScalars* d_sc = nullptr;
    double* d_part_s = nullptr;
    int* d_part_b = nullptr;
    DevScalars* h_sc = nullptr;
    std::vector<MtTensor> tens;  // host copy (pointers and layouts)
    // profiling: events around the two passes of synchronous steps
    bool profiling = false;
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
    neox_profile prof{};
    std::string last_error;
};

namespace {

thread_local std::string g_multi_create_error;

neox_status mfail(neox_multi* h, neox_status st, const std::string& msg) {
    if (h) h->last_error = msg; else g_multi_create_error = msg;
    return st;
}

neox_status mcuda_fail(neox_multi* h, cudaError_t e, const char* what) {
    return mfail(h, e == cudaErrorMemoryAllocation ? NEOX_ERR_OUT_OF_MEMORY : NEOX_ERR_CUDA,
                 std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

void mfree(neox_multi* h) {
    if (h->d_tens) cudaFree(h->d_tens);
    if (h->d_gtab) cudaFree(h->d_gtab);
    if (h->d_seq) cudaFree(h->d_seq);
    if (h->d_odd) cudaFree(h->d_odd);
    if (h->d_sc) cudaFree(h->d_sc);
    if (h->d_part_s) cudaFree(h->d_part_s);
    if (h->d_part_b) cudaFree(h->d_part_b);
    if (h->h_sc) cudaFreeHost(h->h_sc);
    for (auto& ev : h->ev)
        if (ev) cudaEventDestroy(ev);
}

// Pointer table and layout of every tensor; returns an error message or "".
std::string build_tables(const neox_tensor_set* set, std::vector<MtTensor>& tens, std::vector<const uint16_t*>& gtab) {
    const int K = set->num_grads;
    tens.resize(set->ntensors);
    gtab.assign((size_t)set->ntensors * K, nullptr);
    for (int ti = 0; ti < set->ntensors; ti++) {
        const neox_tensor& d = set->tensors[ti];
        MtTensor& T = tens[ti];
        T = MtTensor{};
        T.numel = d.numel;
        T.wd = d.weight_decay;
        T.gbase = ti * K;
        if (!finite(d.weight_decay)) return "tensor " + std::to_string(ti) + ": weight decay must be finite";
        if (d.numel == 0) continue;
        if (!d.master || !d.exp_avg || !d.exp_avg_sq || !d.params || !d.grads)
            return "tensor " + std::to_string(ti) + ": master/exp_avg/exp_avg_sq/params/grads must be non-NULL";
        if (((uintptr_t)d.master | (uintptr_t)d.exp_avg | (uintptr_t)d.exp_avg_sq) & 3u)
            return "tensor " + std::to_string(ti) + ": FP32 arrays must be 4-byte aligned";
        if ((uintptr_t)d.params & 1u) return "tensor " + std::to_string(ti) + ": params must be 2-byte aligned";
        uintptr_t a16[kMaxGrads + 1];
        for (int k = 0; k < K; k++) {
            if (!d.grads[k] || ((uintptr_t)d.grads[k] & 1u))
                return "tensor " + std::to_string(ti) + ": grads[" + std::to_string(k) + "] NULL or misaligned";
            gtab[(size_t)ti * K + k] = static_cast<const uint16_t*>(d.grads[k]);
            a16[k] = (uintptr_t)d.grads[k];
        }
        a16[K] = (uintptr_t)d.params;
        const uintptr_t a32[3] = {(uintptr_t)d.master, (uintptr_t)d.exp_avg, (uintptr_t)d.exp_avg_sq};
        int vec = 1;
        const Layout L = choose_layout(d.numel, a16, K + 1, a32, 3, vec);
        T.master = d.master;
        T.m = d.exp_avg;
        T.v = d.exp_avg_sq;
        T.w = static_cast<uint16_t*>(d.params);
        T.head = L.head;
        T.nvec = L.nvec;
        T.vec = vec;
    }
    return "";
}

// Pass 1's sequence table (tensors with VEC = 8, in order) and the list of
// the other non-empty tensors, from the tensor table and the gradient table.
void build_sequence(const std::vector<MtTensor>& tens, const std::vector<const uint16_t*>& gtab, int K,
                    std::vector<MtSeq>& seq, std::vector<int>& seq_tensor, std::vector<int>& odd,
                    unsigned long long& total8) {
    seq.clear();
    seq_tensor.clear();
    odd.clear();
    total8 = 0;
    for (int ti = 0; ti < (int)tens.size(); ti++) {
        const MtTensor& T = tens[ti];
        if (T.numel == 0 || T.nvec == 0) continue;
        if (T.vec != 8) {
            odd.push_back(ti);
            continue;
        }
        MtSeq e{};
        e.off0 = (long long)T.head - 8ll * (long long)total8;
        total8 += T.nvec;
        e.end = total8;
        e.g0 = gtab[(size_t)ti * K];
        e.gbase = ti * K;
        e.wd = T.wd;
        e.master = T.master;
        e.w = T.w;
        seq.push_back(e);
        seq_tensor.push_back(ti);
    }
}

// Resident-grid size for the multi-tensor kernels (at most one vector of all
// the tensors' vectors per thread).
template <class Kern>
int mt_grid(Kern kernel, int threads, unsigned long long total_vecs, int sm_count, int cap) {
    unsigned long long g = (unsigned long long)sm_count * occupancy(kernel, threads);
    const unsigned long long want = (total_vecs + threads - 1) / threads;
    if (g > want) g = want;
    if (g > (unsigned long long)cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

neox_status mt_enqueue(neox_multi* h, float lr, const float* lr_dev, cudaStream_t st, bool device_bc,
                       neox_step_result* result, bool timed = false) {
    if (!lr_dev && (!finite(lr) || lr < 0.0f)) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "lr must be finite and >= 0");
    if (result && ((uintptr_t)result & 7u)) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "result must be 8-byte aligned");
    if (lr_dev && ((uintptr_t)lr_dev & 3u)) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "lr_device must be 4-byte aligned");
    ScalerArgs sa;
    AdamArgs a;
    make_step_args(h->hp, h->K, lr, h->t, device_bc, sa, a);
    sa.lr_ptr = lr_dev;
    sa.result = result;

    cudaError_t e;
    if (timed && (e = cudaEventRecord(h->ev[0], st)) != cudaSuccess) return mcuda_fail(h, e, "cudaEventRecord");
    {
        auto k1 = h->gdtype == NEOX_FP16 ? mt_stats_kernel<F16> : mt_stats_kernel<BF16>;
        const int grid = h->grid1;
        k1<<<grid, kMtThreads1, 0, st>>>(h->d_tens, h->ntensors, h->d_seq, h->total8, h->d_odd, h->nodd, h->d_gtab,
                                         h->K, sa, h->d_part_s, h->d_part_b, h->d_sc);
        if ((e = cudaGetLastError()) != cudaSuccess) return mcuda_fail(h, e, "pass-1 launch");
        h->prof.launches += 1;
    }
    if (timed && (e = cudaEventRecord(h->ev[1], st)) != cudaSuccess) return mcuda_fail(h, e, "cudaEventRecord");
    if (h->numel > 0) {
        const bool sgd = h->hp.optimizer == NEOX_SGD;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(sgd ? h->grid2_sgd : h->grid2);
        cfg.blockDim = dim3(kMtThreads3);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const MtTensor* tens = h->d_tens;
        const uint16_t* const* gtab = h->d_gtab;
        if (sgd) {
            DevScalars* sc = h->d_sc;
            const MtSeq* seq = h->d_seq;
            const int* odd = h->d_odd;
            const unsigned long long total8 = h->total8;
            e = cudaLaunchKernelEx(&cfg, mt_sgd_kernel_for(h->gdtype, h->wdtype), tens, h->ntensors, seq, total8, odd,
                                   h->nodd, gtab, h->K, a, sc);
        } else {
            DevScalars* sc = h->d_sc;
            const unsigned long long total = h->total_vecs;
            e = cudaLaunchKernelEx(&cfg, mt_adam_kernel_for(h->gdtype, h->wdtype), tens, h->ntensors, gtab, h->K, a, sc,
                                   total);
        }
        if (e != cudaSuccess) return mcuda_fail(h, e, "pass-2 launch");
        h->prof.launches += 1;
    }
    if (timed && (e = cudaEventRecord(h->ev[2], st)) != cudaSuccess) return mcuda_fail(h, e, "cudaEventRecord");
    return NEOX_OK;
}

neox_status mt_refresh(neox_multi* h) {
    if (!h->async_used) return NEOX_OK;
    DeviceGuard g(h->device);
    cudaError_t e;
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return mcuda_fail(h, e, "waiting for asynchronous steps");
    DevScalars r;
    if ((e = cudaMemcpy(&r, h->d_sc, sizeof(r), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return mcuda_fail(h, e, "reading the device scaler state");
    h->scale = r.scale;
    h->good = r.good;
    h->t = r.t;
    return NEOX_OK;
}

}  // namespace

extern "C" {

neox_status neox_multi_create(const neox_tensor_set* set, const neox_hparams* hp, int device, neox_multi** out) {
    g_multi_create_error.clear();
    if (!out) return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "out is NULL");
    if (!set) return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "tensor set is NULL");
    if (const char* why = check_hparams(hp)) return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, why);
    if (set->ntensors < 0 || (set->ntensors > 0 && !set->tensors))
        return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "ntensors must be >= 0 with a tensor array");
    if (set->num_grads < 1 || set->num_grads > kMaxGrads)
        return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "num_grads must be in [1, 64]");
    if ((set->wdtype != NEOX_FP16 && set->wdtype != NEOX_BF16) || (set->gdtype != NEOX_FP16 && set->gdtype != NEOX_BF16))
        return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "dtype must be NEOX_FP16 or NEOX_BF16");
    std::vector<MtTensor> tens;
    std::vector<const uint16_t*> gtab;
    const std::string why = build_tables(set, tens, gtab);
    if (!why.empty()) return mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, why);

    auto* h = new (std::nothrow) neox_multi();
    if (!h) return mfail(nullptr, NEOX_ERR_OUT_OF_MEMORY, "host allocation failed");
    h->device = device;
    h->ntensors = set->ntensors;
    h->K = set->num_grads;
    h->wdtype = set->wdtype;
    h->gdtype = set->gdtype;
    h->hp = *hp;
    h->scale = hp->init_scale;
    for (const auto& T : tens) {
        h->numel += T.numel;
        h->total_vecs += T.nvec;
    }
    neox_status st = NEOX_OK;
    cudaError_t e;
    {
        int ndev = 0;
        if ((e = cudaGetDeviceCount(&ndev)) != cudaSuccess) { st = mcuda_fail(nullptr, e, "cudaGetDeviceCount"); goto done; }
        if (device < 0 || device >= ndev) { st = mfail(nullptr, NEOX_ERR_INVALID_ARGUMENT, "no such CUDA device"); goto done; }
        DeviceGuard g(device);
        if (!g.ok) { st = mfail(nullptr, NEOX_ERR_CUDA, "cudaSetDevice failed"); goto done; }
        int major = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess) {
            st = mcuda_fail(nullptr, e, "cudaDeviceGetAttribute");
            goto done;
        }
        if (major != 10) { st = mfail(nullptr, NEOX_ERR_UNSUPPORTED, "this library is built for sm_100a (B200)"); goto done; }
        h->max_parts = h->sm_count * kMaxBlocksPerSm;
        const size_t nt = tens.size() ? tens.size() : 1, ng = gtab.size() ? gtab.size() : 1;
        if ((e = cudaMalloc(&h->d_tens, sizeof(MtTensor) * nt)) != cudaSuccess ||
            (e = cudaMalloc((void**)&h->d_gtab, sizeof(void*) * ng)) != cudaSuccess ||
            (e = cudaMalloc(&h->d_sc, sizeof(DevScalars))) != cudaSuccess ||
            (e = cudaMalloc(&h->d_part_s, sizeof(double) * h->max_parts)) != cudaSuccess ||
            (e = cudaMalloc(&h->d_part_b, sizeof(int) * h->max_parts)) != cudaSuccess ||
            (e = cudaMallocHost(&h->h_sc, sizeof(DevScalars))) != cudaSuccess ||
            (e = cudaEventCreate(&h->ev[0])) != cudaSuccess || (e = cudaEventCreate(&h->ev[1])) != cudaSuccess ||
            (e = cudaEventCreate(&h->ev[2])) != cudaSuccess) {
            st = mcuda_fail(nullptr, e, "allocation");
            goto done;
        }
        DevScalars init{};
        init.scale = hp->init_scale;
        init.scale_used = hp->init_scale;
        init.hyst = hyst_full(*hp);
        if ((e = cudaMemcpy(h->d_sc, &init, sizeof(init), cudaMemcpyHostToDevice)) != cudaSuccess) {
            st = mcuda_fail(nullptr, e, "cudaMemcpy scalars");
            goto done;
        }
        // Both update passes' grids are set here (set_hparams may switch the
        // rule).  The SGD pass takes its work in chunks of the sequence.
        const MtAdamKernel k2 = mt_adam_kernel_for(h->gdtype, h->wdtype);
        const MtSgdKernel k2s = mt_sgd_kernel_for(h->gdtype, h->wdtype);
        int occ = 0, occ_sgd = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k2, kMtThreads3, 0)) != cudaSuccess ||
            (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_sgd, k2s, kMtThreads3, 0)) != cudaSuccess) {
            st = mcuda_fail(nullptr, e, "configuring the update kernel");
            goto done;
        }
        const unsigned long long want2 = (h->total_vecs + kMtThreads3 - 1) / kMtThreads3;
        unsigned long long g2 = (unsigned long long)h->sm_count * (occ < 1 ? 1 : occ);
        unsigned long long g2s = (unsigned long long)h->sm_count * (occ_sgd < 1 ? 1 : occ_sgd);
        if (g2 > want2) g2 = want2;
        if (g2s > want2) g2s = want2;
        h->grid2 = g2 < 1 ? 1 : (int)g2;
        h->grid2_sgd = g2s < 1 ? 1 : (int)g2s;
        auto k1 = h->gdtype == NEOX_FP16 ? mt_stats_kernel<F16> : mt_stats_kernel<BF16>;
        h->grid1 = mt_grid(k1, kMtThreads1, h->total_vecs, h->sm_count, h->max_parts);
        unsigned long long before = 0;
        for (auto& T : tens) {
            T.before = before;
            before += T.nvec;
        }
        h->tens = tens;
        std::vector<MtSeq> seq;
        std::vector<int> odd;
        build_sequence(tens, gtab, h->K, seq, h->seq_tensor, odd, h->total8);
        h->nseq = (int)seq.size();
        h->nodd = (int)odd.size();
        if ((e = cudaMalloc(&h->d_seq, sizeof(MtSeq) * (seq.empty() ? 1 : seq.size()))) != cudaSuccess ||
            (e = cudaMalloc(&h->d_odd, sizeof(int) * (odd.empty() ? 1 : odd.size()))) != cudaSuccess ||
            (!seq.empty() && (e = cudaMemcpy(h->d_seq, seq.data(), sizeof(MtSeq) * seq.size(),
                                             cudaMemcpyHostToDevice)) != cudaSuccess) ||
            (!odd.empty() && (e = cudaMemcpy(h->d_odd, odd.data(), sizeof(int) * odd.size(),
                                             cudaMemcpyHostToDevice)) != cudaSuccess)) {
            st = mcuda_fail(nullptr, e, "copying the sequence table");
            goto done;
        }
        if ((!tens.empty() && (e = cudaMemcpy(h->d_tens, tens.data(), sizeof(MtTensor) * tens.size(),
                                              cudaMemcpyHostToDevice)) != cudaSuccess) ||
            (!gtab.empty() && (e = cudaMemcpy(h->d_gtab, gtab.data(), sizeof(void*) * gtab.size(),
                                              cudaMemcpyHostToDevice)) != cudaSuccess)) {
            st = mcuda_fail(nullptr, e, "copying the tensor tables");
            goto done;
        }
    }
done:
    if (st != NEOX_OK) {
        DeviceGuard g(device);
        mfree(h);
        delete h;
        return st;
    }
    *out = h;
    return NEOX_OK;
}

void neox_multi_destroy(neox_multi* h) {
    if (!h) return;
    {
        DeviceGuard g(h->device);
        mfree(h);
    }
    delete h;
}

const char* neox_multi_last_error(const neox_multi* h) {
    return h ? h->last_error.c_str() : g_multi_create_error.c_str();
}

neox_status neox_multi_rebind_grads(neox_multi* h, const void* const* grads) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (!grads && h->ntensors > 0) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "grads is NULL");
    std::vector<const uint16_t*> gtab((size_t)h->ntensors * h->K, nullptr);
    for (int ti = 0; ti < h->ntensors; ti++) {
        const MtTensor& T = h->tens[ti];
        if (T.numel == 0) continue;
        for (int k = 0; k < h->K; k++) {
            const void* p = grads[(size_t)ti * h->K + k];
            // the new pointers must keep the tensor's vector layout
            const int al = 2 * T.vec;
            if (!p || (((uintptr_t)p + 2 * T.head) % al) != 0 || ((uintptr_t)p & 1u))
                return mfail(h, NEOX_ERR_INVALID_ARGUMENT,
                             "tensor " + std::to_string(ti) + ": grads[" + std::to_string(k) +
                                 "] NULL or with another alignment than at create");
            gtab[(size_t)ti * h->K + k] = static_cast<const uint16_t*>(p);
        }
    }
    std::vector<MtSeq> seq;
    std::vector<int> seq_tensor, odd;
    unsigned long long total8 = 0;
    build_sequence(h->tens, gtab, h->K, seq, seq_tensor, odd, total8);  // same layout: only g0 changes
    DeviceGuard g(h->device);
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && !gtab.empty())
        e = cudaMemcpy(h->d_gtab, gtab.data(), sizeof(void*) * gtab.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !seq.empty())
        e = cudaMemcpy(h->d_seq, seq.data(), sizeof(MtSeq) * seq.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return mcuda_fail(h, e, "updating the gradient table");
    return NEOX_OK;
}

neox_status neox_multi_step(neox_multi* h, float lr, void* cuda_stream, neox_step_result* out) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->last_error.clear();
    if (!out) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "out is NULL");
    DeviceGuard g(h->device);
    if (!g.ok) return mfail(h, NEOX_ERR_CUDA, "cudaSetDevice failed");
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (neox_status s = mt_enqueue(h, lr, nullptr, st, h->async_used, nullptr, h->profiling); s != NEOX_OK) return s;
    cudaError_t e;
    if ((e = cudaMemcpyAsync(h->h_sc, h->d_sc, sizeof(DevScalars), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return mcuda_fail(h, e, "cudaMemcpyAsync result");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return mcuda_fail(h, e, "step execution");
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

neox_status neox_multi_set_profiling(neox_multi* h, int32_t enable) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->profiling = enable != 0;
    return NEOX_OK;
}

neox_status neox_multi_get_profile(const neox_multi* h, neox_profile* out) {
    if (!h || !out) return NEOX_ERR_INVALID_ARGUMENT;
    *out = h->prof;
    return NEOX_OK;
}

neox_status neox_multi_reset_profile(neox_multi* h) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    const int64_t launches = h->prof.launches;
    h->prof = neox_profile{};
    h->prof.launches = launches;
    return NEOX_OK;
}

neox_status neox_multi_step_async(neox_multi* h, float lr, const float* lr_device, void* cuda_stream,
                                  neox_step_result* result) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    h->last_error.clear();
    DeviceGuard g(h->device);
    if (!g.ok) return mfail(h, NEOX_ERR_CUDA, "cudaSetDevice failed");
    h->async_used = true;
    return mt_enqueue(h, lr, lr_device, static_cast<cudaStream_t>(cuda_stream), true, result);
}

neox_status neox_multi_set_hparams(neox_multi* h, const neox_hparams* hp) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (const char* why = check_hparams(hp)) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, why);
    h->hp = *hp;
    return NEOX_OK;
}

neox_status neox_multi_get_state(const neox_multi* h, float* scale, int32_t* good, int64_t* t) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (neox_status s = mt_refresh(const_cast<neox_multi*>(h)); s != NEOX_OK) return s;
    if (scale) *scale = h->scale;
    if (good) *good = h->good;
    if (t) *t = h->t;
    return NEOX_OK;
}

neox_status neox_multi_set_state(neox_multi* h, float scale, int32_t good, int64_t t) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.0f) || !finite(scale) || good < 0 || t < 0)
        return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "state needs a finite scale > 0, good >= 0, t >= 0");
    DeviceGuard g(h->device);
    cudaError_t e = cudaSuccess;
    if (h->async_used) e = cudaDeviceSynchronize();
    DevScalars s{};
    s.scale = scale;
    s.scale_used = scale;
    s.good = good;
    s.t = t;
    s.hyst = hyst_full(h->hp);
    if (e == cudaSuccess) e = cudaMemcpy(h->d_sc, &s, sizeof(s), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return mcuda_fail(h, e, "writing the scaler state");
    h->scale = scale;
    h->good = good;
    h->t = t;
    return NEOX_OK;
}

neox_status neox_multi_get_hysteresis(const neox_multi* h, int32_t* count) {
    if (!h || !count) return NEOX_ERR_INVALID_ARGUMENT;
    DeviceGuard g(h->device);
    cudaError_t e = h->async_used ? cudaDeviceSynchronize() : cudaSuccess;
    if (e == cudaSuccess) e = cudaMemcpy(count, &h->d_sc->hyst, sizeof(int32_t), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? NEOX_OK : mcuda_fail(const_cast<neox_multi*>(h), e, "reading the hysteresis count");
}

neox_status neox_multi_set_hysteresis(neox_multi* h, int32_t count) {
    if (!h) return NEOX_ERR_INVALID_ARGUMENT;
    if (count < 0) return mfail(h, NEOX_ERR_INVALID_ARGUMENT, "the hysteresis count must be >= 0");
    DeviceGuard g(h->device);
    cudaError_t e = h->async_used ? cudaDeviceSynchronize() : cudaSuccess;
    if (e == cudaSuccess) e = cudaMemcpy(&h->d_sc->hyst, &count, sizeof(int32_t), cudaMemcpyHostToDevice);
    return e == cudaSuccess ? NEOX_OK : mcuda_fail(h, e, "writing the hysteresis count");
}

}  // extern "C"
