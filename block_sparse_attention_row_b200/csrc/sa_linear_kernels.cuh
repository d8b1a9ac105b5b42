// sa_linear_kernels.cuh - the linear branch of the sparse + linear
// combination: feature maps and per-head linear-attention state.
//
// Method: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
// (gist.science summary) §2A: O = alpha * O_s + (1 - alpha) * O_l, O_s the
// sparse attention over a row's kept key blocks and O_l linear attention over
// the rest of the row. Readings (the page prints no feature map): phi(x) =
// elu(x) + 1, and O_l(t) = phi(q_t)^T H_c / phi(q_t)^T z_c over the complement
// tokens c of the row. Computed without forming the complement:
//   H_c = H - sum over kept blocks of phi(K_j)^T V_j,   z_c = z - sum phi(K_j)
// with H = phi(K)^T V and z = sum_u phi(k_u) over all valid keys of the head.
// The kept sums are taken by the attention kernel's linear variant; this file
// holds
//   phi_kernel          phi(Q), phi(K) in bf16 (the operands of every product
//                       of the branch, so the kept and total sums use the
//                       same rounded features), and per key block the fp32
//                       sum of its phi(k) rows;
//   lin_state_kernel    H = phi(K)^T V per head on the tensor cores, over a
//                       split of the tokens (fp32 partial sums per split);
//   lin_finalize_kernel sums the splits and the block sums in a fixed order
//                       and writes H as a bf16 pair (hi, lo = H - hi) and z.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"
#include "sa_attn_kernel.cuh"

namespace sa {
namespace lin {

using attn::Desc;
using attn::desc_at;
using attn::desc_split;
using attn::mnmajor_desc;

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(fminf(x, 0.f)); }

// One CTA per 64-token block of one head (blockIdx.x < 2 * n_b: the first
// n_b are Q blocks, the rest K blocks; blockIdx.y = b*H + h), 128 threads,
// 16-byte loads. K blocks also write zpart[bh, j, c] = sum of the block's
// bf16-rounded phi(k) (fp32, rows in order).
template <int D>
__global__ void __launch_bounds__(128)
phi_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, __nv_bfloat16* __restrict__ pQ,
           __nv_bfloat16* __restrict__ pK, float* __restrict__ zpart, int N, int n_b) {
    constexpr int CG = D / 8, RG = 128 / CG;
    __shared__ float red[RG][D];
    const int bh = blockIdx.y;
    int blk = blockIdx.x;
    const bool isk = blk >= n_b;
    if (isk) blk -= n_b;
    const int lo = blk * 64;
    const int valid = min(64, N - lo);
    const size_t base = ((size_t)bh * N + lo) * D;
    const uint4* src = reinterpret_cast<const uint4*>((isk ? K : Q) + base);
    uint4* dst = reinterpret_cast<uint4*>((isk ? pK : pQ) + base);
    const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int r = rg; r < valid; r += RG) {
        const uint4 v = __ldg(src + (size_t)r * CG + cg);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            o[e] = pack_bf16x2(phi(__uint_as_float(w[e] << 16)), phi(__uint_as_float(w[e] & 0xFFFF0000u)));
            acc[2 * e] += __uint_as_float(o[e] << 16);
            acc[2 * e + 1] += __uint_as_float(o[e] & 0xFFFF0000u);
        }
        dst[(size_t)r * CG + cg] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (!isk) return;
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rg][cg * 8 + e] = acc[e];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += 128) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) s += red[g][c];
        zpart[((size_t)bh * n_b + blk) * D + c] = s;
    }
}

// H partial sums: CTA (bh, sp) covers the 128-token chunks [c0, c1) of head
// bh and writes hpart[bh, sp] = sum over its tokens of phi(k)^T v (fp32, D x
// D, row c = channel of phi(k), column c' = channel of v). Warp 0 lane 0
// loads the chunks by TMA (two stages), warp 1 lane 0 issues the products
// D[c][c'] += A[c][t] B[c'][t] with A = phi(K) chunk and B = V chunk, both
// MN-major (channels contiguous), accumulating in TMEM; then all four warps
// read the accumulator (one TMEM lane quarter each).
constexpr int LS_THREADS = 128;
constexpr int LS_CHUNK = 128;

template <int D>
struct LSLayout {
    static constexpr int SLABS = D / 64;
    static constexpr int CHUNK_BYTES = LS_CHUNK * D * 2;
    static constexpr int NST = 2;
    static constexpr int OFF_CTRL = NST * 2 * CHUNK_BYTES;
    static constexpr int DYN_BYTES = OFF_CTRL + 256 + 1024;
};

struct LSCtrl {
    uint64_t full[2], empty[2], done;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(LS_THREADS, 1)
lin_state_kernel(const __grid_constant__ CUtensorMap tmPK, const __grid_constant__ CUtensorMap tmV,
                 float* __restrict__ hpart, int n_chunks, int splits, unsigned long long lim) {
    static_assert(D == 128, "the linear state is built for d = 128 (M = 128 channels)");
    using L = LSLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    LSCtrl& C = *reinterpret_cast<LSCtrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.x, sp = blockIdx.y;
    const int c0 = (int)((long long)n_chunks * sp / splits), c1 = (int)((long long)n_chunks * (sp + 1) / splits);
    if (threadIdx.x == 0) {
        for (int s = 0; s < L::NST; ++s) {
            mbar_init(&C.full[s], 1);
            mbar_init(&C.empty[s], 1);
        }
        mbar_init(&C.done, 1);
        C.abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&C.tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = C.tmem_base;
    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            int n = 0;
            for (int c = c0; ok && c < c1; ++c, ++n) {
                const int s = n % L::NST;
                if (n >= L::NST &&
                    !mbar_wait_bounded(&C.empty[s], ((n / L::NST) - 1) & 1, abort_flag, 0xA001, lim)) {
                    ok = false;
                    break;
                }
                uint8_t* a = smem + s * 2 * L::CHUNK_BYTES;
                mbar_arrive_expect_tx(&C.full[s], 2 * L::CHUNK_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl) {
                    tma_load_3d(a + sl * (LS_CHUNK * 128), &tmPK, &C.full[s], sl * 64, c * LS_CHUNK, bh);
                    tma_load_3d(a + L::CHUNK_BYTES + sl * (LS_CHUNK * 128), &tmV, &C.full[s], sl * 64, c * LS_CHUNK, bh);
                }
            }
            if (!ok)
                for (int m = (n > L::NST ? n - L::NST : 0); m < n; ++m)
                    for (uint64_t t0 = globaltimer_ns();
                         !mbar_try_wait(&C.full[m % L::NST], (m / L::NST) & 1) && globaltimer_ns() - t0 < lim;) {
                    }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // A = phi(K) chunk: element (m = c, k = t) at t * D + c: MN-major.
            // B = V chunk: element (n = c', k = t) at t * D + c': MN-major.
            constexpr uint32_t IDESC = make_idesc_bf16(128, D, true) | (1u << 15);
            const Desc a_desc = desc_split(mnmajor_desc(smem_u32(smem), LS_CHUNK * 128));
            const Desc b_desc = desc_split(mnmajor_desc(smem_u32(smem + L::CHUNK_BYTES), LS_CHUNK * 128));
            int n = 0;
            for (int c = c0; ok && c < c1; ++c, ++n) {
                const int s = n % L::NST;
                if (!mbar_wait_spin(&C.full[s], (n / L::NST) & 1, abort_flag, 0xA002, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t so = (uint32_t)(s * 2 * L::CHUNK_BYTES) >> 4;
#pragma unroll
                for (int kk = 0; kk < LS_CHUNK / 16; ++kk) {
                    const uint32_t ko = (uint32_t)(kk * 16 * 128) >> 4;
                    umma_ss(tmem, desc_at(a_desc, so + ko), desc_at(b_desc, so + ko), IDESC, (n | kk) ? 1u : 0u);
                }
                umma_commit(&C.empty[s]);
            }
            umma_commit(&C.done);
        }
    }
    __syncwarp();
    // Every warp: wait for the last product, then store its 32 rows.
    const bool w = mbar_wait_bounded(&C.done, 0, abort_flag, 0xA003, lim);
    tc_fence_after();
    if (__all_sync(0xFFFFFFFFu, w) && c1 > c0) {
        const int row = warp * 32 + lane;
        uint32_t v[64];
        float* out = hpart + (((size_t)bh * splits + sp) * D + row) * D;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            tmem_ld64(tmem + ((uint32_t)(warp * 32) << 16) + h * 64, v);
            float4* o4 = reinterpret_cast<float4*>(out + h * 64);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                o4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                    __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
    } else if (c1 <= c0) {
        const int row = warp * 32 + lane;
        float4* o4 = reinterpret_cast<float4*>(hpart + (((size_t)bh * splits + sp) * D + row) * D);
        for (int e = 0; e < D / 4; ++e) o4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// H = sum of the splits (in order), z = sum of the block sums (in order);
// H is written as hi = bf16(H), lo = bf16(H - hi), row-major [c][c'] (the
// layout of a V tile: the B operand of the attention kernel's total product).
// One CTA per head, D threads.
template <int D>
__global__ void __launch_bounds__(D)
lin_finalize_kernel(const float* __restrict__ hpart, const float* __restrict__ zpart, __nv_bfloat16* __restrict__ Hhi,
                    __nv_bfloat16* __restrict__ Hlo, float* __restrict__ z, int splits, int n_b) {
    const int bh = blockIdx.x, c = threadIdx.x;
    for (int r = 0; r < D; ++r) {
        float h = 0.f;
        for (int sp = 0; sp < splits; ++sp) h += hpart[(((size_t)bh * splits + sp) * D + r) * D + c];
        const __nv_bfloat16 hi = __float2bfloat16_rn(h);
        const size_t o = ((size_t)bh * D + r) * D + c;
        Hhi[o] = hi;
        Hlo[o] = __float2bfloat16_rn(h - __bfloat162float(hi));
    }
    float s = 0.f;
    for (int j = 0; j < n_b; ++j) s += zpart[((size_t)bh * n_b + j) * D + c];
    z[(size_t)bh * D + c] = s;
}

}  // namespace lin
}  // namespace sa

namespace sa {
namespace lin {

// ------------------------------------------------------------ combination
// sparse_linear_kernel: per query-block row (bh, i) with kept list idx[0:cnt]:
//   O_acc = phi(Q_i) H - sum over kept tiles of (phi(Q_i) phi(K_t)^T) V_t
//   l     = sum over kept tiles of rowsum(phi(Q_i) phi(K_t)^T)
//   O_l   = O_acc / (phi(q) . z - l), or 0 when every key block is kept
//   O     = alpha * O_s + (1 - alpha) * O_l
// One row pipeline per CTA, rows interleaved over the CTAs. 192 threads:
// warps 0-3 the elementwise step and epilogue (one query row per thread,
// one TMEM lane), warp 4 the TMA producer, warp 5 the tcgen05 issuer.
// TMEM: S double-buffered [0, 128) and [128, 256) (the kept tile's
// negated weights, bf16, are written back over its first 64 columns and
// read by the P V product), O [256, 256 + d). The products of tile t+1 run
// while the weights of tile t are formed; the total product phi(Q) H (as
// hi + lo bf16 parts) is added into the same accumulator after the last
// tile, so the subtraction happens in fp32 inside the tensor core.
constexpr int SL_THREADS = 192;
constexpr int SL_PRODUCER = 4, SL_MMA = 5;
constexpr int SL_MROWS = 128, SL_TILE = 128, SL_BK = 64;

template <int D>
struct SLLayout {
    static constexpr int SLABS = D / 64;
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE_BYTES;            // 2 slots
    static constexpr int OFF_V = 3 * TILE_BYTES;        // 2 slots
    static constexpr int OFF_H = 5 * TILE_BYTES;        // hi, lo
    static constexpr int OFF_CTRL = 7 * TILE_BYTES;
    static constexpr int DYN_BYTES = OFF_CTRL + 512 + 1024;
    static_assert(DYN_BYTES <= 232448, "shared memory budget");
};

struct SLCtrl {
    uint64_t q_full, q_empty, k_full[2], k_empty[2], v_full[2], v_empty[2], h_full, h_empty;
    uint64_t s_full[2], p_full[2], o_full, acc_free, drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct SLParams {
    const int32_t* cnt;        // [rows]
    const int32_t* idx;        // [rows, n_k]
    const __nv_bfloat16* pQ;   // phi(Q) [BH, N, D] bf16
    const float* z;            // [BH, D]
    const void* Os;            // the sparse branch's output [BH, N, D] (o_dtype)
    const float* alpha;        // [BH, N]
    void* O;                   // [BH, N, D] (o_dtype)
    int N, n_q, n_k, rows, out_f32;
    unsigned long long wait_limit_ns;
};

enum SLSite : unsigned int {
    SL_W_Q = 0xB101, SL_W_QE = 0xB102, SL_W_K = 0xB103, SL_W_KE = 0xB104, SL_W_V = 0xB105, SL_W_VE = 0xB106,
    SL_W_H = 0xB107, SL_W_HE = 0xB108, SL_W_S = 0xB109, SL_W_P = 0xB10A, SL_W_O = 0xB10B, SL_W_ACC = 0xB10C
};

__device__ __forceinline__ int sl_count(const SLParams& prm, int r) {
    int c = __ldg(prm.cnt + r);
    if (c < 0 || c > prm.n_k) {
        record_error(SA_STATUS_DEVICE_ASSERT, 0xC000u);
        c = c < 0 ? 0 : prm.n_k;
    }
    return c;
}
__device__ __forceinline__ int sl_entry(const SLParams& prm, int r, int c, int e) {
    if (e >= c) return -1;
    const int j = __ldg(prm.idx + (size_t)r * prm.n_k + e);
    if (j < 0 || j >= prm.n_k) {
        record_error(SA_STATUS_DEVICE_ASSERT, 0xB000u);
        return -1;
    }
    return j;
}

template <int D, int BQ>
__global__ void __launch_bounds__(SL_THREADS, 1)
sparse_linear_kernel(const __grid_constant__ CUtensorMap tmPQ, const __grid_constant__ CUtensorMap tmPK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmHhi,
                     const __grid_constant__ CUtensorMap tmHlo, const SLParams prm) {
    static_assert(D == 128, "the sparse + linear kernel is built for d = 128");
    using L = SLLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SLCtrl& C = *reinterpret_cast<SLCtrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_k = prm.n_k;
    const uint64_t lim = prm.wait_limit_ns;
    // Rows interleaved over the CTAs (r = blockIdx.x + k gridDim.x): at any time
    // the grid works on one or two heads, whose phi(K) and V stay in L2.
    const int r_begin = blockIdx.x, r_end = prm.rows, r_step = gridDim.x;

    if (threadIdx.x == 0) {
        mbar_init(&C.q_full, 1);
        mbar_init(&C.q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&C.k_full[i], 1);
            mbar_init(&C.k_empty[i], 1);
            mbar_init(&C.v_full[i], 1);
            mbar_init(&C.v_empty[i], 1);
            mbar_init(&C.s_full[i], 1);
            mbar_init(&C.p_full[i], 4);
        }
        mbar_init(&C.h_full, 1);
        mbar_init(&C.h_empty, 1);
        mbar_init(&C.o_full, 1);
        mbar_init(&C.acc_free, 4);
        mbar_init(&C.drain, 1);
        C.abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == SL_MMA) {
        tmem_alloc(&C.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = C.tmem_base;

    if (warp == SL_PRODUCER) {
        // -------------------------------------------------------- producer
        int g = 0, kq = 0, gk = 0, gv = 0;
        bool ok = true;
        for (int r = r_begin; ok && r < r_end; r += r_step) {
            const int cnt = sl_count(prm, r);
            const int nt = (cnt + 1) / 2;
            const int bh = r / prm.n_q, qb = r % prm.n_q;
            if (kq > 0 && (!wait_warp(&C.q_empty, (kq - 1) & 1, abort_flag, SL_W_QE, lim) ||
                           !wait_warp(&C.h_empty, (kq - 1) & 1, abort_flag, SL_W_HE, lim))) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&C.q_full, L::TILE_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl)
                    tma_load_3d(smem + L::OFF_Q + sl * (SL_MROWS * 128), &tmPQ, &C.q_full, sl * 64, qb * BQ, bh);
                mbar_arrive_expect_tx(&C.h_full, 2 * L::TILE_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl) {
                    tma_load_3d(smem + L::OFF_H + sl * (128 * 128), &tmHhi, &C.h_full, sl * 64, 0, bh);
                    tma_load_3d(smem + L::OFF_H + L::TILE_BYTES + sl * (128 * 128), &tmHlo, &C.h_full, sl * 64, 0, bh);
                }
            }
            ++kq;
            int window = -1;
            for (int t = 0; t < nt; ++t, ++g) {
                const int e0 = 2 * t;
                if ((e0 & 31) == 0) window = sl_entry(prm, r, cnt, e0 + lane);
                const int j0 = __shfl_sync(0xFFFFFFFFu, window, e0 & 31);
                const int j1 = __shfl_sync(0xFFFFFFFFu, window, (e0 + 1) & 31);
                const int r0 = (j0 >= 0 ? j0 : n_k) * SL_BK;   // absent: a row past N, zeros
                const int r1 = (j1 >= 0 ? j1 : n_k) * SL_BK;
                const int sk = g & 1;
                if (g >= 2 && !wait_warp(&C.k_empty[sk], ((g >> 1) - 1) & 1, abort_flag, SL_W_KE, lim)) { ok = false; break; }
                if (lane == 0) {
                    uint8_t* dst = smem + L::OFF_K + sk * L::TILE_BYTES;
                    mbar_arrive_expect_tx(&C.k_full[sk], L::TILE_BYTES);
                    for (int sl = 0; sl < L::SLABS; ++sl) {
                        tma_load_3d(dst + sl * (SL_TILE * 128), &tmPK, &C.k_full[sk], sl * 64, r0, bh);
                        tma_load_3d(dst + sl * (SL_TILE * 128) + SL_BK * 128, &tmPK, &C.k_full[sk], sl * 64, r1, bh);
                    }
                }
                gk = g + 1;
                if (g >= 2 && !wait_warp(&C.v_empty[sk], ((g >> 1) - 1) & 1, abort_flag, SL_W_VE, lim)) { ok = false; break; }
                if (lane == 0) {
                    uint8_t* dst = smem + L::OFF_V + sk * L::TILE_BYTES;
                    mbar_arrive_expect_tx(&C.v_full[sk], L::TILE_BYTES);
                    for (int sl = 0; sl < L::SLABS; ++sl) {
                        tma_load_3d(dst + sl * (SL_TILE * 128), &tmV, &C.v_full[sk], sl * 64, r0, bh);
                        tma_load_3d(dst + sl * (SL_TILE * 128) + SL_BK * 128, &tmV, &C.v_full[sk], sl * 64, r1, bh);
                    }
                }
                gv = g + 1;
            }
        }
        if (*abort_flag && lane == 0) {
            if (kq > 0) {
                drain_wait(&C.q_full, (kq - 1) & 1, lim);
                drain_wait(&C.h_full, (kq - 1) & 1, lim);
            }
            for (int gg = (gk > 2 ? gk - 2 : 0); gg < gk; ++gg) drain_wait(&C.k_full[gg & 1], (gg >> 1) & 1, lim);
            for (int gg = (gv > 2 ? gv - 2 : 0); gg < gv; ++gg) drain_wait(&C.v_full[gg & 1], (gg >> 1) & 1, lim);
        }
    } else if (warp == SL_MMA) {
        // ---------------------------------------------------------- issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = make_idesc_bf16(SL_MROWS, SL_TILE, false);
            constexpr uint32_t IDESC_O = make_idesc_bf16(SL_MROWS, D, true);
            const Desc q_desc = desc_split(attn::kmajor_desc(smem_u32(smem + L::OFF_Q)));
            const Desc k_desc = desc_split(attn::kmajor_desc(smem_u32(smem + L::OFF_K)));
            const Desc v_desc = desc_split(mnmajor_desc(smem_u32(smem + L::OFF_V), SL_TILE * 128));
            const Desc h_desc = desc_split(mnmajor_desc(smem_u32(smem + L::OFF_H), 128 * 128));
            const uint32_t tO = tmem + 256;   // S buffers at tmem + 128 * (tile & 1)
            int g = 0, kq = 0, rown = 0;
            bool ok = true;
            auto issue_s = [&](int gt) -> bool {
                const int sk = gt & 1;
                if (!mbar_wait_spin(&C.k_full[sk], (gt >> 1) & 1, abort_flag, SL_W_K, lim)) return false;
                tc_fence_after();
                const uint32_t ko = (uint32_t)(sk * L::TILE_BYTES) >> 4;
#pragma unroll
                for (int sl = 0; sl < L::SLABS; ++sl)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t o = (sl * (SL_MROWS * 128) + kk * 32) >> 4;
                        umma_ss(tmem + 128u * sk, desc_at(q_desc, o), desc_at(k_desc, ko + o), IDESC_S, (sl | kk) ? 1u : 0u);
                    }
                umma_commit(&C.s_full[sk]);
                umma_commit(&C.k_empty[sk]);
                return true;
            };
            for (int r = r_begin; ok && r < r_end; r += r_step) {
                const int nt = (sl_count(prm, r) + 1) / 2;
                if (!mbar_wait_spin(&C.q_full, kq & 1, abort_flag, SL_W_Q, lim)) { ok = false; break; }
                ++kq;
                if (nt > 0 && !issue_s(g)) { ok = false; break; }
                for (int t = 0; t < nt; ++t) {
                    if (t + 1 < nt && !issue_s(g + 1)) { ok = false; break; }
                    const int sb = g & 1;
                    if (!mbar_wait_spin(&C.p_full[sb], (g >> 1) & 1, abort_flag, SL_W_P, lim) ||
                        !mbar_wait_spin(&C.v_full[sb], (g >> 1) & 1, abort_flag, SL_W_V, lim)) {
                        ok = false;
                        break;
                    }
                    if (t == 0 && rown > 0 && !mbar_wait_spin(&C.acc_free, (rown - 1) & 1, abort_flag, SL_W_ACC, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t vo = (uint32_t)(sb * L::TILE_BYTES) >> 4;
#pragma unroll
                    for (int kk = 0; kk < SL_TILE / 16; ++kk)
                        umma_ts(tO, tmem + 128u * sb + 8 * kk, desc_at(v_desc, vo + ((kk * 16 * 128) >> 4)), IDESC_O,
                                (t > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&C.v_empty[sb]);
                    ++g;
                }
                if (!ok) break;
                // The total: O += phi(Q_i) (H_hi + H_lo).
                if (!mbar_wait_spin(&C.h_full, (kq - 1) & 1, abort_flag, SL_W_H, lim) ||
                    (nt == 0 && rown > 0 && !mbar_wait_spin(&C.acc_free, (rown - 1) & 1, abort_flag, SL_W_ACC, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ao = ((kk >> 2) * (SL_MROWS * 128) + (kk & 3) * 32) >> 4;
                        const uint32_t bo = (part * L::TILE_BYTES + kk * 16 * 128) >> 4;
                        umma_ss(tO, desc_at(q_desc, ao), desc_at(h_desc, bo), IDESC_O,
                                (nt > 0 || part > 0 || kk > 0) ? 1u : 0u);
                    }
                umma_commit(&C.h_empty);
                umma_commit(&C.q_empty);
                umma_commit(&C.o_full);
                ++rown;
            }
            if (!ok) {
                umma_commit(&C.drain);
                drain_wait(&C.drain, 0, lim);
            }
        }
    } else {
        // ------------------------------------------- weights and epilogue
        const int wq = warp;                      // warps 0-3: TMEM lane quarter
        const int row = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tO = tmem + 256 + lane_off;   // S buffers at tmem + lane_off + 128 * (tile & 1)
        const bool f32 = prm.out_f32 != 0;
        int g = 0, rown = 0;
        bool ok = true;
        for (int r = r_begin; ok && r < r_end; r += r_step) {
            const int cnt = sl_count(prm, r);
            const int nt = (cnt + 1) / 2;
            const int bh = r / prm.n_q, qb = r % prm.n_q;
            const int q_tok = qb * BQ + row;
            const bool row_valid = row < BQ && q_tok < prm.N;
            const size_t off = ((size_t)bh * prm.N + q_tok) * D;
            // phi(q) . z for this row (its features as the products use them: bf16).
            float qz = 0.f;
            if (row_valid) {
                const uint4* pq = reinterpret_cast<const uint4*>(prm.pQ + off);
                const float4* z4 = reinterpret_cast<const float4*>(prm.z + (size_t)bh * D);
#pragma unroll 4
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 v = __ldg(pq + c);
                    const float4 za = __ldg(z4 + 2 * c), zb = __ldg(z4 + 2 * c + 1);
                    qz = fmaf(__uint_as_float(v.x << 16), za.x, qz);
                    qz = fmaf(__uint_as_float(v.x & 0xFFFF0000u), za.y, qz);
                    qz = fmaf(__uint_as_float(v.y << 16), za.z, qz);
                    qz = fmaf(__uint_as_float(v.y & 0xFFFF0000u), za.w, qz);
                    qz = fmaf(__uint_as_float(v.z << 16), zb.x, qz);
                    qz = fmaf(__uint_as_float(v.z & 0xFFFF0000u), zb.y, qz);
                    qz = fmaf(__uint_as_float(v.w << 16), zb.z, qz);
                    qz = fmaf(__uint_as_float(v.w & 0xFFFF0000u), zb.w, qz);
                }
            }
            float l = 0.f;                         // sum of the kept (bf16) weights
            int window = -1;
            for (int t = 0; t < nt; ++t, ++g) {
                const int e0 = 2 * t;
                if ((e0 & 31) == 0) window = sl_entry(prm, r, cnt, e0 + lane);
                const int j0 = __shfl_sync(0xFFFFFFFFu, window, e0 & 31);
                const int j1 = __shfl_sync(0xFFFFFFFFu, window, (e0 + 1) & 31);
                const int v0 = j0 < 0 ? 0 : min(SL_BK, prm.N - j0 * SL_BK);
                const int v1 = j1 < 0 ? 0 : min(SL_BK, prm.N - j1 * SL_BK);
                const int sb = g & 1;
                if (!wait_warp(&C.s_full[sb], (g >> 1) & 1, abort_flag, SL_W_S, lim)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tS = tmem + lane_off + 128u * sb;
                uint32_t s[128];
                tmem_ld128(tS, s);
                uint32_t pk[64];
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const int c0 = 2 * c, c1 = 2 * c + 1;
                    const bool ok0 = c0 < 64 ? c0 < v0 : c0 - 64 < v1;
                    const bool ok1 = c1 < 64 ? c1 < v0 : c1 - 64 < v1;
                    const float w0 = ok0 ? __uint_as_float(s[c0]) : 0.f;
                    const float w1 = ok1 ? __uint_as_float(s[c1]) : 0.f;
                    const uint32_t p = pack_bf16x2(w0, w1);
                    acc0 += __uint_as_float(p << 16);
                    acc1 += __uint_as_float(p & 0xFFFF0000u);
                    pk[c] = p ^ 0x80008000u;        // the negated weights (exact in bf16)
                }
                l += acc0 + acc1;
                tmem_st64_nowait(tS, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&C.p_full[sb]);
            }
            if (!ok) break;
            if (!wait_warp(&C.o_full, rown & 1, abort_flag, SL_W_O, lim)) { ok = false; break; }
            tc_fence_after();
            uint32_t o[D];
            tmem_ld128(tO, o);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&C.acc_free);
            ++rown;
            if (!row_valid) continue;
            // O_l = complement numerator / complement weight; none when every block is kept.
            const float den = qz - l;
            const float inv = (cnt < n_k && den > 0.f) ? 1.f / den : 0.f;
            const float a = __ldg(prm.alpha + (size_t)bh * prm.N + q_tok);
            const float b = (1.f - a) * inv;
            if (f32) {
                const float4* os = reinterpret_cast<const float4*>(static_cast<const float*>(prm.Os) + off);
                float4* out = reinterpret_cast<float4*>(static_cast<float*>(prm.O) + off);
#pragma unroll
                for (int e = 0; e < D / 4; ++e) {
                    const float4 x = __ldg(os + e);
                    out[e] = make_float4(fmaf(a, x.x, b * __uint_as_float(o[4 * e])),
                                         fmaf(a, x.y, b * __uint_as_float(o[4 * e + 1])),
                                         fmaf(a, x.z, b * __uint_as_float(o[4 * e + 2])),
                                         fmaf(a, x.w, b * __uint_as_float(o[4 * e + 3])));
                }
            } else {
                const uint4* os = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(prm.Os) + off);
                uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.O) + off);
#pragma unroll
                for (int e = 0; e < D / 8; ++e) {
                    const uint4 x = __ldg(os + e);
                    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
                    uint32_t y[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        y[q] = pack_bf16x2(fmaf(a, __uint_as_float(xs[q] << 16), b * __uint_as_float(o[8 * e + 2 * q])),
                                           fmaf(a, __uint_as_float(xs[q] & 0xFFFF0000u),
                                                b * __uint_as_float(o[8 * e + 2 * q + 1])));
                    out[e] = make_uint4(y[0], y[1], y[2], y[3]);
                }
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == SL_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace lin
}  // namespace sa
