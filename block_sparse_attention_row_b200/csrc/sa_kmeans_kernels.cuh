// sa_kmeans_kernels.cuh - semantic-aware permutation of the tokens ahead of
// the block-sparse path: k-means of one head's token vectors, the stable
// permutation by cluster, and row gathers and scatters.
//
// Method: "Sparse VideoGen2: Accelerate Video Generation with Sparse
// Attention via Semantic-Aware Permutation" (gist.science summary) §2A: Q and
// K tokens are clustered independently by k-means and reordered so that each
// cluster is contiguous; consistent permutations of Q rows and of K, V rows
// leave dense attention unchanged, and the output is restored to token order.
// §2C starts k-means from cached centroids (the `init` argument here).
// Every decision is taken in stated fp32 arithmetic so that the result is
// exact (the page names no initialisation, distance or tie rule):
//   distance  sum over channels, in order, of (x_j - m_j)^2, the subtraction,
//             the product and each addition rounded to fp32 (no fused
//             multiply-add); the nearest centroid wins, ties to the lower index;
//   centroid  fp32 sum of the members in ascending token order / member count;
//             an empty cluster keeps its centroid;
//   order     tokens sorted by cluster, ascending token order within one.
// Kernels, per (batch, head):
//   km_init_kernel     centroids = the tokens at floor(c N / C);
//   km_assign_kernel   one thread per token, centroids staged in shared memory;
//   km_sort_kernel     one CTA per head: counting sort over up to 8 warps
//                      token ranges, stable by token order (cluster offsets
//                      for the update, the permutation);
//   km_update_kernel   one thread per (cluster, channel): sequential sums;
//   permute_rows_kernel  Y[i] = X[perm[i]] or Y[perm[i]] = X[i].
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"

namespace sa {
namespace km {

constexpr int AS_THREADS = 128;     // tokens per CTA of the assignment
constexpr int AS_CHUNK = 32;        // centroids staged per pass

template <int D>
__global__ void __launch_bounds__(D)
km_init_kernel(const __nv_bfloat16* __restrict__ X, float* __restrict__ M, int N, int C) {
    const int c = blockIdx.x, bh = blockIdx.y, j = threadIdx.x;
    const long long t = (long long)c * N / C;
    M[((size_t)bh * C + c) * D + j] = __bfloat162float(X[((size_t)bh * N + t) * D + j]);
}

// Four centroids at a time (independent accumulators); strict < keeps the
// lower index on ties, since centroids are visited in ascending order.
template <int D>
__global__ void __launch_bounds__(AS_THREADS)
km_assign_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ M, int32_t* __restrict__ ids,
                 int N, int C) {
    __shared__ __align__(16) float ms[AS_CHUNK * D];
    const int bh = blockIdx.y;
    const int t = blockIdx.x * AS_THREADS + threadIdx.x;
    const bool valid = t < N;
    float x[D];
    if (valid) {
        const uint4* src = reinterpret_cast<const uint4*>(X + ((size_t)bh * N + t) * D);
#pragma unroll
        for (int q = 0; q < D / 8; ++q) {
            const uint4 v = __ldg(src + q);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
                x[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < D; ++j) x[j] = 0.f;
    }
    float best = INFINITY;
    int best_c = 0;
    const float* Mh = M + (size_t)bh * C * D;
    for (int c0 = 0; c0 < C; c0 += AS_CHUNK) {
        const int nc = min(AS_CHUNK, C - c0);
        __syncthreads();
        // 16-byte loads, several in flight per thread (one L2 round trip per chunk).
        const float4* src = reinterpret_cast<const float4*>(Mh + (size_t)c0 * D);
        float4* dst = reinterpret_cast<float4*>(ms);
#pragma unroll 8
        for (int e = threadIdx.x; e < nc * (D / 4); e += AS_THREADS) dst[e] = __ldg(src + e);
        __syncthreads();
        int c = 0;
        for (; c + 4 <= nc; c += 4) {
            // Four centroids, their channels read 4 at a time (16-byte broadcast
            // loads): the fp32 pipe, not instruction issue, bounds the loop.
            const float4* m4 = reinterpret_cast<const float4*>(ms + c * D);
            float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < D / 4; ++j4) {
                const float4 q0 = m4[j4], q1 = m4[D / 4 + j4], q2 = m4[2 * (D / 4) + j4], q3 = m4[3 * (D / 4) + j4];
                const float c0[4] = {q0.x, q0.y, q0.z, q0.w}, c1[4] = {q1.x, q1.y, q1.z, q1.w};
                const float c2[4] = {q2.x, q2.y, q2.z, q2.w}, c3[4] = {q3.x, q3.y, q3.z, q3.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * j4 + e;
                    const float a0 = __fsub_rn(x[j], c0[e]), a1 = __fsub_rn(x[j], c1[e]);
                    const float a2 = __fsub_rn(x[j], c2[e]), a3 = __fsub_rn(x[j], c3[e]);
                    d0 = __fadd_rn(d0, __fmul_rn(a0, a0));
                    d1 = __fadd_rn(d1, __fmul_rn(a1, a1));
                    d2 = __fadd_rn(d2, __fmul_rn(a2, a2));
                    d3 = __fadd_rn(d3, __fmul_rn(a3, a3));
                }
            }
            if (d0 < best) { best = d0; best_c = c0 + c; }
            if (d1 < best) { best = d1; best_c = c0 + c + 1; }
            if (d2 < best) { best = d2; best_c = c0 + c + 2; }
            if (d3 < best) { best = d3; best_c = c0 + c + 3; }
        }
        for (; c < nc; ++c) {
            const float* m0 = ms + c * D;
            float d0 = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) {
                const float a0 = __fsub_rn(x[j], m0[j]);
                d0 = __fadd_rn(d0, __fmul_rn(a0, a0));
            }
            if (d0 < best) { best = d0; best_c = c0 + c; }
        }
    }
    if (valid) ids[(size_t)bh * N + t] = best_c;
}

// One CTA per head, W = blockDim.x / 32 warps, warp w taking the w-th
// contiguous range of the tokens: per-warp histograms of the cluster ids
// (shared memory), an exclusive scan of the totals into the cluster offsets,
// per-warp cursors (a cluster's offset plus the counts of the warps before),
// then each warp places its tokens in ascending order, 32 at a time: lanes
// with the same id (match) take consecutive positions in lane order and
// their group's leader advances the cursor. The order within a cluster is
// therefore the token order. off gets the C + 1 cluster offsets (off[C] = N).
// Shared memory: (W + 1) * C ints.
__global__ void __launch_bounds__(256)
km_sort_kernel(const int32_t* __restrict__ ids, int32_t* __restrict__ perm, int32_t* __restrict__ off, int N, int C) {
    extern __shared__ int32_t sort_smem[];
    const int W = blockDim.x / 32;
    const int bh = blockIdx.x, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    int32_t* tot = sort_smem;                    // [C]: totals, then cluster offsets
    int32_t* cur = sort_smem + C + warp * C;     // [C]: this warp's counts, then cursors
    const int32_t* id = ids + (size_t)bh * N;
    int32_t* pm = perm + (size_t)bh * N;
    int32_t* of = off + (size_t)bh * (C + 1);
    const int span = (N + W - 1) / W;
    const int t_lo = min(N, warp * span), t_hi = min(N, t_lo + span);
    for (int e = threadIdx.x; e < (W + 1) * C; e += blockDim.x) sort_smem[e] = 0;
    __syncthreads();
    for (int t = t_lo + lane; t < t_hi; t += 32) atomicAdd(&cur[id[t]], 1);
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int s = 0;
        for (int w = 0; w < W; ++w) s += sort_smem[C + w * C + c];
        tot[c] = s;
    }
    __syncthreads();
    if (warp == 0) {
        int run = 0;   // exclusive scan, 32 clusters at a time
        for (int c0 = 0; c0 < C; c0 += 32) {
            const int c = c0 + lane;
            const int v = c < C ? tot[c] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            if (c < C) {
                tot[c] = run + incl - v;
                of[c] = run + incl - v;
            }
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) of[C] = run;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int run = tot[c];
        for (int w = 0; w < W; ++w) {
            int32_t* h = sort_smem + C + w * C + c;
            const int n = *h;
            *h = run;
            run += n;
        }
    }
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    for (int base = t_lo; base < t_hi; base += 32) {
        const int t = base + lane;
        const bool valid = t < t_hi;
        const int c = valid ? id[t] : -1 - lane;   // invalid lanes match nobody
        const uint32_t grp = __match_any_sync(0xFFFFFFFFu, c);
        if (valid) pm[cur[c] + __popc(grp & lt)] = t;
        __syncwarp();
        if (valid && (grp & lt) == 0) cur[c] += __popc(grp);
        __syncwarp();
    }
}

// Warps of km_sort_kernel for C clusters: as many as (W + 1) * C ints of
// shared memory allow within `budget` bytes, at most 8.
inline int km_sort_warps(int C, size_t budget) {
    long long w = (long long)(budget / (4 * (size_t)C)) - 1;
    return (int)(w < 1 ? 1 : (w > 8 ? 8 : w));
}

// One CTA per (cluster, head), one thread per channel: the members are
// perm[off[c] .. off[c + 1]) in ascending token order; their channel values
// are added in that order in fp32 and divided by the count.
template <int D>
__global__ void __launch_bounds__(D)
km_update_kernel(const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm,
                 const int32_t* __restrict__ off, float* __restrict__ M, int N, int C) {
    const int c = blockIdx.x, bh = blockIdx.y, j = threadIdx.x;
    const int32_t* of = off + (size_t)bh * (C + 1);
    const int a = of[c], b = of[c + 1];
    if (b <= a) return;                       // empty: the centroid stays
    const int32_t* pm = perm + (size_t)bh * N;
    const __nv_bfloat16* Xh = X + (size_t)bh * N * D;
    float s = 0.f;
    for (int i = a; i < b; ++i) s = __fadd_rn(s, __bfloat162float(Xh[(size_t)pm[i] * D + j]));
    M[((size_t)bh * C + c) * D + j] = __fdiv_rn(s, (float)(b - a));
}

// Rows of [BH, N, D] elements of ESIZE bytes (2: bf16, 4: fp32): inverse = 0
// gathers Y[i] = X[perm[i]], inverse = 1 scatters Y[perm[i]] = X[i]. Each
// row is ROW_BYTES / 16 lanes, one 16-byte chunk each (a warp moves 1, 2 or
// 4 rows at once). An entry outside [0, N) is recorded as a device
// assertion and its row is skipped.
template <int ROW_BYTES>
struct PermuteShape {
    static constexpr int LANES = ROW_BYTES / 16;          // lanes per row
    static constexpr int ROWS_PER_WARP = 32 / LANES;
    static constexpr int ROWS_PER_CTA = 8 * ROWS_PER_WARP;   // 256 threads
    static_assert(LANES >= 1 && LANES <= 32 && 32 % LANES == 0, "row of 16..512 bytes");
};

template <int ROW_BYTES>
__global__ void __launch_bounds__(256)
permute_rows_kernel(const uint8_t* __restrict__ X, const int32_t* __restrict__ perm, uint8_t* __restrict__ Y, int N,
                    int inverse) {
    using S = PermuteShape<ROW_BYTES>;
    const int bh = blockIdx.y;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int i = blockIdx.x * S::ROWS_PER_CTA + warp * S::ROWS_PER_WARP + lane / S::LANES;
    const int c = lane % S::LANES;
    if (i >= N) return;
    const int p = perm[(size_t)bh * N + i];
    if (p < 0 || p >= N) {                    // not a permutation entry: reported, row skipped
        if (c == 0) record_error(SA_STATUS_DEVICE_ASSERT, 0x9E00u);
        return;
    }
    const int src = inverse ? i : p, dst = inverse ? p : i;
    const uint4* s = reinterpret_cast<const uint4*>(X + ((size_t)bh * N + src) * ROW_BYTES);
    uint4* d = reinterpret_cast<uint4*>(Y + ((size_t)bh * N + dst) * ROW_BYTES);
    d[c] = __ldg(s + c);
}

}  // namespace km
}  // namespace sa
