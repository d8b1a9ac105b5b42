// sa_mask_kernels.cuh - steps 1-3 of the path: block pooling, block scores,
// and the per-row hybrid Top-k + Top-p selection.
//
// Method: "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
// Masking and Distillation Fine-Tuning" (gist.science summary) §1 Problem
// Statement (Top-k and Top-p rules) and §2A Hybrid Top-k + Top-p Masking
// (per-row union); block scores from pooled queries and keys as in "SLA2:
// Sparse-Linear Attention with Learnable Routing and QAT" §2B and mean
// pooling of contiguous blocks as in "Sparse VideoGen2" §1.
//
// Three kernels, each sized for its own bound:
//   pool_kernel    HBM-bound: reads Q and K once (16-byte loads), writes the
//                  fp32 block means Qbar [BH, n_q, d] and Kbar [BH, n_k, d].
//   score_kernel   fp32 CUDA-core GEMM per head: logits = Qbar Kbar^T/sqrt(d)
//                  into an [BH*n_q, ld] scratch matrix (stays mostly in L2).
//   select_kernel  one warp per score row: softmax (from logits) or a given
//                  P, then the exact selection described below.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"

namespace sa {
namespace mask {

constexpr int POOL_THREADS = 128;

// Mean of the valid tokens of one query block or key block. blockIdx.x in
// [0, n_q) pools a Q block, [n_q, n_q + n_k) a K block; blockIdx.y = b*H + h.
template <int D>
__global__ void __launch_bounds__(POOL_THREADS)
pool_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
            float* __restrict__ Qbar, float* __restrict__ Kbar, int N, int bq, int bk, int n_q,
            int n_k) {
    constexpr int CG = D / 8;              // 16-byte chunks per token row
    constexpr int RG = POOL_THREADS / CG;  // token rows read in parallel
    __shared__ float red[RG][D];

    const int bh = blockIdx.y;
    int blk = blockIdx.x;
    const __nv_bfloat16* X;
    float* out;
    int bs;
    if (blk < n_q) {
        X = Q;
        out = Qbar + ((size_t)bh * n_q + blk) * D;
        bs = bq;
    } else {
        blk -= n_q;
        X = K;
        out = Kbar + ((size_t)bh * n_k + blk) * D;
        bs = bk;
    }
    const int lo = blk * bs;
    const int valid = min(N - lo, bs);
    const uint4* src = reinterpret_cast<const uint4*>(X + ((size_t)bh * N + lo) * D);
    const int cg = threadIdx.x % CG;
    const int rg = threadIdx.x / CG;

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 8
    for (int r = rg; r < valid; r += RG) {
        const uint4 v = __ldg(src + (size_t)r * CG + cg);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[2 * e] += __uint_as_float(w[e] << 16);
            acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rg][cg * 8 + e] = acc[e];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += POOL_THREADS) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) s += red[g][c];
        out[c] = s / (float)valid;
    }
}

// logits[bh*n_q + i][j] = scale * sum_c Qbar[bh,i,c] * Kbar[bh,j,c], fp32.
// CTA tile: 32 query blocks x 64 key blocks, channels in chunks of 64; each
// thread accumulates 2 x 4 outputs.
constexpr int SC_TI = 32, SC_TJ = 64, SC_TC = 64, SC_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(SC_THREADS)
score_kernel(const float* __restrict__ Qbar, const float* __restrict__ Kbar,
             float* __restrict__ logits, int ld, int n_q, int n_k, float scale) {
    __shared__ __align__(16) float qs[SC_TI][SC_TC + 4];
    __shared__ __align__(16) float kt[SC_TC][SC_TJ];

    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * SC_TI;
    const int j0 = blockIdx.x * SC_TJ;
    const int t = threadIdx.x;
    const float* qsrc = Qbar + (size_t)bh * n_q * D;
    const float* ksrc = Kbar + (size_t)bh * n_k * D;
    const int tr = t / 16, tj = t % 16;
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};

    for (int c0 = 0; c0 < D; c0 += SC_TC) {
        // Q tile, row-major (float4 along channels, coalesced).
        for (int e = t; e < SC_TI * (SC_TC / 4); e += SC_THREADS) {
            const int r = e / (SC_TC / 4), c4 = e % (SC_TC / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i0 + r < n_q)
                v = *reinterpret_cast<const float4*>(qsrc + (size_t)(i0 + r) * D + c0 + 4 * c4);
            *reinterpret_cast<float4*>(&qs[r][4 * c4]) = v;
        }
        // K tile, transposed to [channel][key] so that consecutive threads
        // read consecutive keys below.
        for (int e = t; e < SC_TJ * (SC_TC / 4); e += SC_THREADS) {
            const int j = e % SC_TJ, c4 = e / SC_TJ;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j0 + j < n_k)
                v = *reinterpret_cast<const float4*>(ksrc + (size_t)(j0 + j) * D + c0 + 4 * c4);
            kt[4 * c4 + 0][j] = v.x;
            kt[4 * c4 + 1][j] = v.y;
            kt[4 * c4 + 2][j] = v.z;
            kt[4 * c4 + 3][j] = v.w;
        }
        __syncthreads();
#pragma unroll 4
        for (int c = 0; c < SC_TC; c += 4) {
            const float4 q0 = *reinterpret_cast<const float4*>(&qs[2 * tr][c]);
            const float4 q1 = *reinterpret_cast<const float4*>(&qs[2 * tr + 1][c]);
            const float q0v[4] = {q0.x, q0.y, q0.z, q0.w};
            const float q1v[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float4 kv = *reinterpret_cast<const float4*>(&kt[c + cc][4 * tj]);
                a0[0] = fmaf(q0v[cc], kv.x, a0[0]);
                a0[1] = fmaf(q0v[cc], kv.y, a0[1]);
                a0[2] = fmaf(q0v[cc], kv.z, a0[2]);
                a0[3] = fmaf(q0v[cc], kv.w, a0[3]);
                a1[0] = fmaf(q1v[cc], kv.x, a1[0]);
                a1[1] = fmaf(q1v[cc], kv.y, a1[1]);
                a1[2] = fmaf(q1v[cc], kv.z, a1[2]);
                a1[3] = fmaf(q1v[cc], kv.w, a1[3]);
            }
        }
        __syncthreads();
    }
    const int jj = j0 + 4 * tj;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int i = i0 + 2 * tr + rr;
        if (i >= n_q) continue;
        const float* a = rr ? a1 : a0;
        float* dst = logits + ((size_t)bh * n_q + i) * ld + jj;
        if (jj + 3 < ld) {
            *reinterpret_cast<float4*>(dst) =
                make_float4(a[0] * scale, a[1] * scale, a[2] * scale, a[3] * scale);
        } else {
            for (int e = 0; e < 4; ++e)
                if (jj + e < ld) dst[e] = a[e] * scale;
        }
    }
}

// ----------------------------------------------------------- selection
__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Fixed-point mass of one score: floor(P * 2^31). P in [0, 1] so the fp32
// product is exact and the truncating conversion is exact.
__device__ __forceinline__ uint64_t fixed_mass(uint32_t bits) {
    return __float2ull_rz(__uint_as_float(bits) * 2147483648.0f);
}

// Boundary search over one score row held as fp32 bit patterns (P >= 0, so
// unsigned order is numeric order). For the metric "fixed-point mass"
// (MASS = true) or "number of entries" (MASS = false) it finds the largest
// 31-bit value v such that the metric summed over the entries >= v still
// reaches `target`, most significant bit first. The entries still able to
// decide the answer (those inside the current range [v, v | (2^(b+1) - 1)])
// are kept in `work` and compacted in place after every bit, so each step
// only touches the survivors. Returns v and, through the out-parameters, the
// count and mass of the entries strictly above v. Integer sums only: the
// answer does not depend on the order of the reductions.
struct Boundary {
    uint32_t v;
    int n_above;
    uint64_t mass_above;
};

template <bool MASS>
__device__ Boundary boundary_search(const uint32_t* __restrict__ bits, uint32_t* __restrict__ work,
                                    int n, uint64_t target, int lane) {
    for (int j = lane; j < n; j += 32) work[j] = bits[j];
    __syncwarp();
    const uint32_t lt_mask = (1u << lane) - 1u;
    int m = n;
    uint32_t v = 0;
    int n_above = 0;
    uint64_t mass_above = 0;
    for (int b = 30; b >= 0; --b) {
        const uint32_t bit = 1u << b;
        uint64_t hi_mass = 0;
        uint32_t hi_cnt = 0;
        for (int j = lane; j < m; j += 32) {
            const uint32_t x = work[j];
            if (x & bit) {
                ++hi_cnt;
                if (MASS) hi_mass += fixed_mass(x);
            }
        }
        hi_cnt = warp_sum_u32(hi_cnt);
        if (MASS) hi_mass = warp_sum_u64(hi_mass);
        const uint64_t reach = MASS ? mass_above + hi_mass : (uint64_t)(n_above + (int)hi_cnt);
        const bool take = reach >= target;
        if (take) {
            v |= bit;  // entries without this bit fall below v
        } else {
            n_above += (int)hi_cnt;  // entries with this bit lie above the range
            mass_above += hi_mass;
        }
        const int keep_n = take ? (int)hi_cnt : m - (int)hi_cnt;
        if (keep_n != m) {
            int out = 0;
            for (int base = 0; base < m; base += 32) {
                const int j = base + lane;
                uint32_t x = 0;
                bool keep = false;
                if (j < m) {
                    x = work[j];
                    keep = ((x & bit) != 0) == take;
                }
                const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
                __syncwarp();
                if (keep) work[out + __popc(bal & lt_mask)] = x;
                out += __popc(bal);
                __syncwarp();
            }
            m = keep_n;
        }
    }
    if (!MASS) mass_above = 0;
    return {v, n_above, mass_above};
}

constexpr int SEL_MAX_WARPS = 4;
constexpr int SEL_SMEM_BUDGET = 200 * 1024;

// Warps (rows) per CTA of select_kernel for a row length n_k: each warp
// holds its row twice in shared memory (8 bytes per entry).
inline int select_warps_per_cta(int n_k) {
    int w = SEL_SMEM_BUDGET / (8 * n_k);
    return w < 1 ? 1 : (w > SEL_MAX_WARPS ? SEL_MAX_WARPS : w);
}

// One warp per score row. The kept set is the first L entries of the order
// "score descending, then index ascending", L = max(kc, m_p):
//   kc  = number of Top-k blocks (computed on the host);
//   m_p = shortest prefix whose fixed-point mass reaches T = ceil(p * W).
// m_p comes from the mass boundary v (entries above v, then as many of the
// entries equal to v as the remaining mass needs); if kc is larger, the
// count boundary of kc is searched the same way. The kept indices are then
// written in ascending order, ties at the boundary taken by lower index.
// The result equals the prefix of a full sort bit for bit.
template <bool FROM_LOGITS>
__global__ void __launch_bounds__(SEL_MAX_WARPS * 32)
select_kernel(const float* __restrict__ in, int ld_in, int n_rows, int n_k, int kc, double p,
              int32_t* __restrict__ cnt, int32_t* __restrict__ idx, uint8_t* __restrict__ mask,
              float* __restrict__ P_out) {
    extern __shared__ uint32_t sel_smem[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int wpc = blockDim.x / 32;
    const long long row = (long long)blockIdx.x * wpc + warp;
    if (row >= n_rows) return;
    uint32_t* bits = sel_smem + (size_t)warp * 2 * n_k;
    uint32_t* work = bits + n_k;
    const float* src = in + (size_t)row * ld_in;

    if (FROM_LOGITS) {
        float mx = -INFINITY;
        for (int j = lane; j < n_k; j += 32) mx = fmaxf(mx, src[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        float sum = 0.f;
        for (int j = lane; j < n_k; j += 32) {
            const float e = expf(src[j] - mx);
            bits[j] = __float_as_uint(e);
            sum += e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        for (int j = lane; j < n_k; j += 32) {
            const float pj = __fdiv_rn(__uint_as_float(bits[j]), sum);
            bits[j] = __float_as_uint(pj);
            if (P_out) P_out[(size_t)row * n_k + j] = pj;
        }
    } else {
        bool bad = false;
        for (int j = lane; j < n_k; j += 32) {
            const uint32_t b = __float_as_uint(src[j]);
            bad |= (b > 0x3F800000u);  // negative, > 1, Inf or NaN
            bits[j] = b;
        }
        if (__any_sync(0xFFFFFFFFu, bad) && lane == 0)
            record_error(SA_STATUS_DEVICE_ASSERT, 0x5E1Eu);
    }
    __syncwarp();

    // L = number of kept entries; (v, n_above) = its boundary score and the
    // number of entries strictly above it.
    int L = kc;
    bool have_boundary = false;
    Boundary bd = {0u, 0, 0ull};
    if (p >= 1.0) {
        L = n_k;
    } else {
        uint64_t w = 0;
        for (int j = lane; j < n_k; j += 32) w += fixed_mass(bits[j]);
        const uint64_t W = warp_sum_u64(w);
        const uint64_t T = (uint64_t)ceil(p * (double)W);
        if (T > 0) {
            const Boundary mb = boundary_search<true>(bits, work, n_k, T, lane);
            const uint64_t wb = fixed_mass(mb.v);  // > 0 for scores in [0, 1]
            const uint64_t need = wb ? (T - mb.mass_above + wb - 1) / wb : 1;
            const int m_p = (int)(mb.n_above + need);
            if (m_p >= kc) {
                L = m_p;
                bd = mb;
                have_boundary = true;
            }
        }
    }
    L = min(L, n_k);

    int32_t* idx_row = idx + (size_t)row * n_k;
    uint8_t* mask_row = mask ? mask + (size_t)row * n_k : nullptr;
    if (L == n_k) {
        for (int j = lane; j < n_k; j += 32) {
            idx_row[j] = j;
            if (mask_row) mask_row[j] = 1;
        }
    } else if (L <= 0) {
        L = 0;
        if (mask_row)
            for (int j = lane; j < n_k; j += 32) mask_row[j] = 0;
    } else {
        if (!have_boundary) bd = boundary_search<false>(bits, work, n_k, (uint64_t)L, lane);
        const uint32_t v = bd.v;
        const int ties_kept = L - bd.n_above;
        int ties_before = 0, kept_before = 0;
        const uint32_t lt_mask = (1u << lane) - 1u;
        for (int base = 0; base < n_k; base += 32) {
            const int j = base + lane;
            const bool in_row = j < n_k;
            const uint32_t b = in_row ? bits[j] : 0u;
            const bool gt = in_row && b > v;
            const bool eq = in_row && b == v;
            const uint32_t eq_ballot = __ballot_sync(0xFFFFFFFFu, eq);
            const int tie_rank = ties_before + __popc(eq_ballot & lt_mask);
            const bool keep = gt || (eq && tie_rank < ties_kept);
            const uint32_t keep_ballot = __ballot_sync(0xFFFFFFFFu, keep);
            if (keep) idx_row[kept_before + __popc(keep_ballot & lt_mask)] = j;
            if (mask_row && in_row) mask_row[j] = keep ? 1 : 0;
            ties_before += __popc(eq_ballot);
            kept_before += __popc(keep_ballot);
        }
    }
    if (lane == 0) cnt[row] = L;
}

}  // namespace mask
}  // namespace sa
