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

// Mean of the valid rows of one block of X (`valid` token rows of D bf16
// channels from `src`), computed by the POOL_THREADS threads of a group
// (tid = 0 .. POOL_THREADS-1) through `red` ([POOL_THREADS / (D / 8)][D]
// floats of shared memory), `sync` being the group's barrier. Each thread
// sums its 16-byte column chunk over the rows tid / (D / 8), + RG, ... in
// order; the partial sums are then added in group order and divided by
// `valid`. Used by pool_kernel and by the single-launch path, so both give
// the same bits.
template <int D, typename Sync>
__device__ __forceinline__ void pool_block(const __nv_bfloat16* __restrict__ src_rows, float* __restrict__ out,
                                           int valid, int tid, float* red, Sync sync) {
    constexpr int CG = D / 8;              // 16-byte chunks per token row
    constexpr int RG = POOL_THREADS / CG;  // token rows read in parallel
    const uint4* src = reinterpret_cast<const uint4*>(src_rows);
    const int cg = tid % CG;
    const int rg = tid / CG;
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
    for (int e = 0; e < 8; ++e) red[rg * D + cg * 8 + e] = acc[e];
    sync();
    for (int c = tid; c < D; c += POOL_THREADS) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) s += red[g * D + c];
        out[c] = s / (float)valid;
    }
}

// Mean of the valid tokens of one query block or key block. blockIdx.x in
// [0, n_q) pools a Q block, [n_q, n_q + n_k) a K block; blockIdx.y = b*H + h.
template <int D>
__global__ void __launch_bounds__(POOL_THREADS)
pool_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
            float* __restrict__ Qbar, float* __restrict__ Kbar, int N, int bq, int bk, int n_q,
            int n_k) {
    __shared__ float red[(POOL_THREADS / (D / 8)) * D];
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
    pool_block<D>(X + ((size_t)bh * N + lo) * D, out, valid, threadIdx.x, red, [] { __syncthreads(); });
}

// logits[bh*n_q + i][j] = scale * sum_c Qbar[bh,i,c] * Kbar[bh,j,c], fp32.
// CTA tile: 64 query blocks x 128 key blocks, channels in chunks of 32 held
// channel-major in shared memory; each of the 256 threads accumulates 4 query
// blocks x 8 key blocks (two groups of 4 adjacent key blocks, 64 apart), so
// one channel step is 32 FMAs for three 16-byte shared-memory loads.
constexpr int SC_TI = 64, SC_TJ = 128, SC_TC = 32, SC_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(SC_THREADS)
score_kernel(const float* __restrict__ Qbar, const float* __restrict__ Kbar,
             float* __restrict__ logits, int ld, int n_q, int n_k, float scale) {
    static_assert(D % SC_TC == 0, "channel chunks");
    __shared__ __align__(16) float qs[SC_TC][SC_TI];
    __shared__ __align__(16) float ks[SC_TC][SC_TJ];

    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * SC_TI;
    const int j0 = blockIdx.x * SC_TJ;
    const int t = threadIdx.x;
    const float* qsrc = Qbar + (size_t)bh * n_q * D;
    const float* ksrc = Kbar + (size_t)bh * n_k * D;
    const int ty = t / 16, tx = t % 16;   // rows 4ty..4ty+3; keys 4tx..4tx+3 and 64+4tx..64+4tx+3
    float acc[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;

    for (int c0 = 0; c0 < D; c0 += SC_TC) {
        // Tiles transposed to [channel][row]. Consecutive threads take
        // consecutive rows, so the transposed shared-memory stores are free of
        // bank conflicts (the 16-byte global reads are then 512 bytes apart).
        for (int e = t; e < SC_TI * (SC_TC / 4); e += SC_THREADS) {
            const int r = e % SC_TI, c4 = e / SC_TI;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i0 + r < n_q) v = *reinterpret_cast<const float4*>(qsrc + (size_t)(i0 + r) * D + c0 + 4 * c4);
            qs[4 * c4 + 0][r] = v.x;
            qs[4 * c4 + 1][r] = v.y;
            qs[4 * c4 + 2][r] = v.z;
            qs[4 * c4 + 3][r] = v.w;
        }
        for (int e = t; e < SC_TJ * (SC_TC / 4); e += SC_THREADS) {
            const int jj = e % SC_TJ, c4 = e / SC_TJ;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j0 + jj < n_k) v = *reinterpret_cast<const float4*>(ksrc + (size_t)(j0 + jj) * D + c0 + 4 * c4);
            ks[4 * c4 + 0][jj] = v.x;
            ks[4 * c4 + 1][jj] = v.y;
            ks[4 * c4 + 2][jj] = v.z;
            ks[4 * c4 + 3][jj] = v.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int c = 0; c < SC_TC; ++c) {
            const float4 a = *reinterpret_cast<const float4*>(&qs[c][4 * ty]);
            const float4 b0 = *reinterpret_cast<const float4*>(&ks[c][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&ks[c][64 + 4 * tx]);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[r][q] = fmaf(av[r], bv[q], acc[r][q]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = i0 + 4 * ty + r;
        if (i >= n_q) continue;
        float* row = logits + ((size_t)bh * n_q + i) * ld;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int jj = j0 + 64 * g + 4 * tx;
            const float* a = &acc[r][4 * g];
            if (jj + 3 < ld) {
                *reinterpret_cast<float4*>(row + jj) = make_float4(a[0] * scale, a[1] * scale, a[2] * scale, a[3] * scale);
            } else {
                for (int e = 0; e < 4; ++e)
                    if (jj + e < ld) row[jj + e] = a[e] * scale;
            }
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
// reaches `target`, most significant bit first. After bit b is decided, the
// entries still able to decide the answer are those that agree with v on the
// bits above b; while there are more than 32 of them each step rescans the row
// and tests that prefix, and once at most 32 are left they are gathered into
// one register per lane and the remaining bits take one ballot each. Returns
// v and, through the out-parameters, the count and mass of the entries
// strictly above v. Integer sums only: the answer does not depend on the
// order of the reductions.
struct Boundary {
    uint32_t v;
    int n_above;
    uint64_t mass_above;
};

template <bool MASS>
__device__ Boundary boundary_search(const uint32_t* __restrict__ bits, const uint64_t* __restrict__ masses,
                                    int n, uint64_t target, int lane) {
    uint32_t v = 0;
    int n_above = 0;
    uint64_t mass_above = 0;
    int m = n;    // entries that agree with v on the bits decided so far
    int b = 30;   // bit 31 is the sign, 0 for every score
    for (; b >= 0 && m > 32; --b) {
        const uint32_t bit = 1u << b;
        uint32_t hi_cnt = 0;
        uint64_t hi_mass = 0;
        for (int j = lane; j < n; j += 32) {
            const uint32_t x = bits[j];
            if ((((x ^ v) >> b) >> 1) == 0u && (x & bit)) {
                ++hi_cnt;
                if (MASS) hi_mass += masses[j];
            }
        }
        hi_cnt = warp_sum_u32(hi_cnt);
        if (MASS) hi_mass = warp_sum_u64(hi_mass);
        const uint64_t reach = MASS ? mass_above + hi_mass : (uint64_t)(n_above + (int)hi_cnt);
        if (reach >= target) {
            v |= bit;  // entries without this bit fall below v
            m = (int)hi_cnt;
        } else {
            n_above += (int)hi_cnt;  // entries with this bit lie above the range
            mass_above += hi_mass;
            m -= (int)hi_cnt;
        }
    }
    if (b >= 0) {
        // At most 32 candidates left: one per lane.
        uint32_t x = 0;
        uint64_t xm = 0;
        int got = 0;
        for (int base = 0; base < n; base += 32) {
            const int j = base + lane;
            const bool cand = j < n && ((((bits[j] ^ v) >> b) >> 1) == 0u);
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cand);
            const uint32_t xj = cand ? bits[j] : 0u;
            const uint64_t mj = (MASS && cand) ? masses[j] : 0ull;
            // Hand candidate number `slot` to lane `slot`.
#pragma unroll 1
            for (uint32_t rest = bal; rest; rest &= rest - 1) {
                const int src = __ffs(rest) - 1;
                const int dst = got + __popc(bal & ((1u << src) - 1u));
                const uint32_t xv = __shfl_sync(0xFFFFFFFFu, xj, src);
                const uint64_t mv = MASS ? __shfl_sync(0xFFFFFFFFu, mj, src) : 0ull;
                if (lane == dst) {
                    x = xv;
                    xm = mv;
                }
            }
            got += __popc(bal);
        }
        bool alive = lane < got;
        for (; b >= 0; --b) {
            const uint32_t bit = 1u << b;
            const bool hi = alive && (x & bit);
            const uint32_t hi_bal = __ballot_sync(0xFFFFFFFFu, hi);
            const uint32_t hi_cnt = __popc(hi_bal);
            const uint64_t hi_mass = MASS ? warp_sum_u64(hi ? xm : 0ull) : 0ull;
            const uint64_t reach = MASS ? mass_above + hi_mass : (uint64_t)(n_above + (int)hi_cnt);
            if (reach >= target) {
                v |= bit;
                alive = hi;
            } else {
                n_above += (int)hi_cnt;
                mass_above += hi_mass;
                alive = alive && !(x & bit);
            }
        }
    }
    if (!MASS) mass_above = 0;
    return {v, n_above, mass_above};
}

constexpr int SEL_MAX_WARPS = 4;
constexpr int SEL_SMEM_BUDGET = 200 * 1024;

// Warps (rows) per CTA of select_kernel for a row length n_k: each warp
// holds its row's score bits and fixed-point masses in shared memory (12
// bytes per entry, rounded up to keep the masses 8-byte aligned).
__host__ __device__ inline int select_row_bytes(int n_k) { return 4 * ((n_k + 1) & ~1) + 8 * n_k; }
inline int select_warps_per_cta(int n_k) {
    int w = SEL_SMEM_BUDGET / select_row_bytes(n_k);
    return w < 1 ? 1 : (w > SEL_MAX_WARPS ? SEL_MAX_WARPS : w);
}

// The selection of one score row by one warp. The kept set is the first L
// entries of the order "score descending, then index ascending",
// L = max(kc, m_p):
//   kc  = number of Top-k blocks (computed on the host);
//   m_p = shortest prefix whose fixed-point mass reaches T = ceil(p * W).
// m_p comes from the mass boundary v (entries above v, then as many of the
// entries equal to v as the remaining mass needs); if kc is larger, the
// count boundary of kc is searched the same way. The kept indices are then
// written in ascending order, ties at the boundary taken by lower index.
// The result equals the prefix of a full sort bit for bit.
// src: the row's logits (FROM_LOGITS: softmax taken here) or scores; bits:
// n_k words of scratch, which may be src itself (each lane rewrites only the
// entries it read); masses: n_k 8-byte words of scratch. Returns L.
template <bool FROM_LOGITS>
__device__ int select_row(const float* src, int n_k, int kc, double p, uint32_t* bits, uint64_t* masses,
                          int32_t* __restrict__ idx_row, uint8_t* __restrict__ mask_row, float* __restrict__ P_row,
                          int lane) {
    if (FROM_LOGITS) {
        float mx = -INFINITY;
        for (int j = lane; j < n_k; j += 32) mx = fmaxf(mx, src[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        // exp(x - max) as 2^((x - max) log2 e) on the MUFU unit (relative error
        // about 2e-7, far below the 1e-6 near-tie scale), and one reciprocal of
        // the sum; P is clamped to 1 so its fixed-point mass stays <= 2^31.
        const float mxl = mx * 1.4426950408889634f;
        float sum = 0.f;
        for (int j = lane; j < n_k; j += 32) {
            const float e = ex2_approx(fmaf(src[j], 1.4426950408889634f, -mxl));
            bits[j] = __float_as_uint(e);
            sum += e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        const float inv = 1.0f / sum;
        for (int j = lane; j < n_k; j += 32) {
            const float pj = fminf(__uint_as_float(bits[j]) * inv, 1.0f);
            bits[j] = __float_as_uint(pj);
            if (P_row) P_row[j] = pj;
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
    } else if (p > 0.0) {
        uint64_t w = 0;
        for (int j = lane; j < n_k; j += 32) {
            const uint64_t mj = fixed_mass(bits[j]);
            masses[j] = mj;
            w += mj;
        }
        const uint64_t W = warp_sum_u64(w);
        const uint64_t T = (uint64_t)ceil(p * (double)W);
        __syncwarp();
        if (T > 0) {
            const Boundary mb = boundary_search<true>(bits, masses, n_k, T, lane);
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
        if (!have_boundary) bd = boundary_search<false>(bits, masses, n_k, (uint64_t)L, lane);
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
    return L;
}

// One warp per score row (select_row above), rows in shared memory.
template <bool FROM_LOGITS>
__global__ void __launch_bounds__(SEL_MAX_WARPS * 32)
select_kernel(const float* __restrict__ in, int ld_in, int n_rows, int n_k, int kc, double p,
              int32_t* __restrict__ cnt, int32_t* __restrict__ idx, uint8_t* __restrict__ mask,
              float* __restrict__ P_out) {
    extern __shared__ __align__(8) unsigned char sel_smem[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int wpc = blockDim.x / 32;
    const long long row = (long long)blockIdx.x * wpc + warp;
    if (row >= n_rows) return;
    uint32_t* bits = reinterpret_cast<uint32_t*>(sel_smem + (size_t)warp * select_row_bytes(n_k));
    uint64_t* masses = reinterpret_cast<uint64_t*>(bits + ((n_k + 1) & ~1));
    const int L = select_row<FROM_LOGITS>(in + (size_t)row * ld_in, n_k, kc, p, bits, masses,
                                          idx + (size_t)row * n_k, mask ? mask + (size_t)row * n_k : nullptr,
                                          P_out ? P_out + (size_t)row * n_k : nullptr, lane);
    if (lane == 0) cnt[row] = L;
}

// ------------------------------------------- single-launch mask phases
// The mask steps run inside the attention kernel's launch (all of its
// threads, before they take their attention roles), separated by grid
// barriers. Each phase computes exactly what pool_kernel, score_kernel and
// select_kernel compute, with the same per-element operation order, so the
// block lists are identical to the three-launch path's.

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier of a cooperative launch: every CTA adds one to *ctr and waits
// until it reaches `target` (CTA count times the barrier's ordinal; the
// counter is zeroed before the launch). The wait is bounded: past `lim` ns
// the CTA records SA_STATUS_TIMEOUT with `site`, sets *abort_flag and goes
// on; a CTA that has given up before arrives without waiting. Returns false
// if this CTA has given up (now or earlier).
__device__ __forceinline__ bool grid_barrier(unsigned int* ctr, unsigned int target, unsigned long long lim,
                                             volatile int* abort_flag, unsigned int site) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);   // arrives even after giving up, so that no other CTA waits on this one
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 0; *abort_flag == 0 && ld_acquire_gpu(ctr) < target; ++it) {
            if ((it & 63u) == 63u && globaltimer_ns() - t0 > lim) {
                record_error(SA_STATUS_TIMEOUT, site);
                *abort_flag = 1;
                break;
            }
        }
        __threadfence();
    }
    __syncthreads();
    return *abort_flag == 0;
}

// Phase A: the block means. Groups of POOL_THREADS threads (a warpgroup
// each, named barrier 1 + group) take (head, block) items in turn, Q blocks
// then K blocks of each head as pool_kernel's grid orders them.
// red: the groups' reduction arrays, (blockDim.x / POOL_THREADS) x
// (POOL_THREADS / (D / 8)) x D floats of shared memory.
template <int D>
__device__ void fused_pool_phase(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                                 float* __restrict__ Qbar, float* __restrict__ Kbar, int BH, int N, int bq, int bk,
                                 int n_q, int n_k, float* red_all) {
    constexpr int RED = (POOL_THREADS / (D / 8)) * D;
    const int grp = threadIdx.x / POOL_THREADS;
    const int ngrp = blockDim.x / POOL_THREADS;
    const int tid = threadIdx.x % POOL_THREADS;
    float* red = red_all + grp * RED;
    auto group_sync = [grp] { asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "n"(POOL_THREADS) : "memory"); };
    const long long per_head = n_q + n_k;
    const long long items = (long long)BH * per_head;
    for (long long it = (long long)blockIdx.x * ngrp + grp; it < items; it += (long long)gridDim.x * ngrp) {
        const int bh = (int)(it / per_head);
        int blk = (int)(it % per_head);
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
        group_sync();   // the group's previous item has read red
        pool_block<D>(X + ((size_t)bh * N + lo) * D, out, min(N - lo, bs), tid, red, group_sync);
    }
}

// Rows of one phase-B item: one per warp of the attention kernel's CTA.
constexpr int FUSED_ROWS = 12;

// Shared memory phase B needs for a row length n_k (pooled query rows,
// logits whose bits the selection overwrites in place, fixed-point masses).
__host__ __device__ inline size_t fused_select_smem(int D, int n_k) {
    const int ldk = (n_k + 3) & ~3;
    return (size_t)FUSED_ROWS * D * 4 + (size_t)FUSED_ROWS * ldk * 4 + (size_t)FUSED_ROWS * n_k * 8;
}

// Phase B: scores and selection, an item being FUSED_ROWS query-block rows
// of one head. The logits of the item's rows against every key block are
// computed as score_kernel computes them (fp32 fused multiply-adds over the
// channels in ascending order from 0, then times `scale`) into shared
// memory; each warp then selects one row (select_row, as select_kernel) and
// writes its kept list and count. Qbar and Kbar were written by other CTAs
// before the grid barrier: they are read through L2 (ld.global.cg).
template <int D>
__device__ void fused_select_phase(const float* __restrict__ Qbar, const float* __restrict__ Kbar, int BH, int n_q,
                                   int n_k, float scale, int kc, double p, int32_t* __restrict__ cnt,
                                   int32_t* __restrict__ idx, uint8_t* smem) {
    const int ldk = (n_k + 3) & ~3;
    float* qs = reinterpret_cast<float*>(smem);                       // [FUSED_ROWS][D]
    float* logit = qs + FUSED_ROWS * D;                               // [FUSED_ROWS][ldk]
    uint64_t* masses = reinterpret_cast<uint64_t*>(logit + FUSED_ROWS * ldk);   // [FUSED_ROWS][n_k]
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nthr = blockDim.x;
    const int tiles = (n_q + FUSED_ROWS - 1) / FUSED_ROWS;
    const long long items = (long long)BH * tiles;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const int bh = (int)(it / tiles);
        const int i0 = (int)(it % tiles) * FUSED_ROWS;
        const int nr = min(FUSED_ROWS, n_q - i0);
        __syncthreads();   // the previous item is done with shared memory
        for (int e = threadIdx.x; e < FUSED_ROWS * (D / 4); e += nthr) {
            const int r = e / (D / 4), c4 = e % (D / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < nr) v = __ldcg(reinterpret_cast<const float4*>(Qbar + ((size_t)bh * n_q + i0 + r) * D) + c4);
            reinterpret_cast<float4*>(qs + r * D)[c4] = v;
        }
        __syncthreads();
        for (int j = threadIdx.x; j < n_k; j += nthr) {
            const float4* kr = reinterpret_cast<const float4*>(Kbar + ((size_t)bh * n_k + j) * D);
            float acc[FUSED_ROWS];
#pragma unroll
            for (int r = 0; r < FUSED_ROWS; ++r) acc[r] = 0.f;
#pragma unroll 4
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 kv = __ldcg(kr + c4);
#pragma unroll
                for (int r = 0; r < FUSED_ROWS; ++r) {
                    const float4 qv = reinterpret_cast<const float4*>(qs + r * D)[c4];
                    acc[r] = fmaf(qv.x, kv.x, acc[r]);
                    acc[r] = fmaf(qv.y, kv.y, acc[r]);
                    acc[r] = fmaf(qv.z, kv.z, acc[r]);
                    acc[r] = fmaf(qv.w, kv.w, acc[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < FUSED_ROWS; ++r)
                if (r < nr) logit[r * ldk + j] = acc[r] * scale;
        }
        __syncthreads();
        if (warp < nr) {
            float* row = logit + warp * ldk;
            const size_t gr = (size_t)bh * n_q + i0 + warp;
            const int L = select_row<true>(row, n_k, kc, p, reinterpret_cast<uint32_t*>(row),
                                           masses + (size_t)warp * n_k, idx + gr * n_k, nullptr, nullptr, lane);
            if (lane == 0) cnt[gr] = L;
        }
    }
}

}  // namespace mask
}  // namespace sa
