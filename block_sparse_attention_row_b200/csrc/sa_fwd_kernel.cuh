// sa_fwd_kernel.cuh - step 4 of the path: block-sparse FlashAttention-style
// forward over the kept (query block, key block) tiles only, for sm_100a.
//
// Method: "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
// Masking and Distillation Fine-Tuning" (gist.science summary) §2C Efficient
// Kernel Implementation: the tensors are split into tiles, the hybrid mask is
// applied per block, and the matmuls and softmax of masked tiles are skipped.
// Here a masked tile is never loaded, multiplied or exponentiated: the CTA
// walks only its row's kept-block list.
//
// One CTA per (b, h, query block); 192 threads in three roles:
//   warp 0      TMA producer: Q once, then K and V of two kept key blocks per
//               128-key tile, gathered by the index list into a 2-stage ring
//               (out-of-range coordinates zero-fill an absent second block);
//   warp 1      tcgen05 issuer (one thread): S = Q K^T into one of two TMEM
//               buffers, O += P V into a TMEM accumulator;
//   warps 2-5   softmax: each thread owns one query row (one TMEM lane),
//               online softmax in base 2 with a lazy rescale of O (only when
//               the running max grows by more than 2^8), P written as bf16
//               into a 128-byte-swizzled shared tile; then the epilogue.
// Tensor-core shapes: S tile M=128 (queries) x N=128 (keys) x K=d; PV tile
// M=128 x N=d x K=128. Both are bf16 x bf16 -> fp32 (kind::f16).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"

namespace sa {
namespace fwd {

constexpr int BK = 64;           // key block (tokens)
constexpr int TILE_N = 128;      // keys per S tile: two kept key blocks
constexpr int MROWS = 128;       // query rows per MMA tile
constexpr int NSTAGE = 2;        // K/V ring depth
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;

// Where a bounded wait gave up (reported in the device error record).
enum WaitSite : unsigned int {
    W_KV_EMPTY = 0xF001, W_Q = 0xF002, W_K_FULL = 0xF003, W_S_FREE = 0xF004,
    W_P_FULL = 0xF005, W_V_FULL = 0xF006, W_S_FULL = 0xF007, W_O_DONE = 0xF008,
    W_META = 0xF009, W_DRAIN = 0xF00A
};

template <int D>
struct SmemLayout {
    static constexpr int SLABS = D / 64;                       // 64-channel (128-byte) slabs
    static constexpr int Q_BYTES = MROWS * D * 2;              // 32 KB at d=128
    static constexpr int KV_BYTES = TILE_N * D * 2;            // per stage, per tensor
    static constexpr int P_BYTES = MROWS * TILE_N * 2;         // 32 KB
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + NSTAGE * KV_BYTES;
    static constexpr int OFF_P = OFF_V + NSTAGE * KV_BYTES;
    static constexpr int OFF_CTRL = OFF_P + P_BYTES;
    static constexpr int CTRL_BYTES = 256;
    // Request enough that only one CTA fits per SM (TMEM_COLS columns each).
    static constexpr int RAW = OFF_CTRL + CTRL_BYTES;
    static constexpr int DYN_BYTES = (RAW < 120 * 1024 ? 120 * 1024 : RAW) + 1024;
};

struct Ctrl {
    uint64_t bar_q;
    uint64_t k_full[NSTAGE];
    uint64_t v_full[NSTAGE];
    uint64_t kv_empty[NSTAGE];
    uint64_t s_full[2];
    uint64_t s_free[2];
    uint64_t p_full;
    uint64_t o_done;
    uint64_t drain;          // abort path: completion of every MMA issued
    int32_t blk[NSTAGE][2];  // key blocks held by a stage (-1 = absent)
    uint32_t tmem_base;
    int abort_flag;
};

struct FwdParams {
    const int32_t* cnt;  // [BH, n_q]
    const int32_t* idx;  // [BH, n_q, n_k]
    __nv_bfloat16* O;    // [BH, N, D]
    float* lse;          // [BH, N] or null
    int N, n_q, n_k, bq;
    int dense;           // 1: every key block, no index list
    float scale_log2;    // log2(e) / sqrt(d)
    unsigned long long wait_limit_ns;
};

// Shared-memory descriptors: 128-byte swizzle, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
    return make_sdesc_sw128(addr, 16u, 1024u);
}
// MN-major B operand (V): 64 channels contiguous per 128-byte row, next 64
// channels `slab_bytes` further on, keys 128 bytes apart, 8-key groups 1024 B.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr, uint32_t slab_bytes) {
    return make_sdesc_sw128(addr, slab_bytes, 1024u);
}

template <int D, int BQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
sparse_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams prm) {
    using L = SmemLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = smem + L::OFF_Q;
    uint8_t* sK = smem + L::OFF_K;
    uint8_t* sV = smem + L::OFF_V;
    uint8_t* sP = smem + L::OFF_P;
    Ctrl& C = *reinterpret_cast<Ctrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int qblk = blockIdx.x;
    const int bh = blockIdx.y;
    const int n_k = prm.n_k;

    // Number of kept key blocks of this row.
    int cnt;
    if (prm.dense) {
        cnt = n_k;
    } else {
        cnt = prm.cnt[(size_t)bh * prm.n_q + qblk];
        if (cnt < 0 || cnt > n_k) {
            if (threadIdx.x == 0) record_error(SA_STATUS_DEVICE_ASSERT, 0xC000u);
            cnt = cnt < 0 ? 0 : n_k;
        }
    }
    const int nt = (cnt + 1) / 2;
    const int32_t* idx_row = prm.dense ? nullptr : prm.idx + ((size_t)bh * prm.n_q + qblk) * n_k;

    if (threadIdx.x == 0) {
        mbar_init(&C.bar_q, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&C.k_full[s], 1);
            mbar_init(&C.v_full[s], 1);
            mbar_init(&C.kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&C.s_full[b], 1);
            mbar_init(&C.s_free[b], 128);
        }
        mbar_init(&C.p_full, 128);
        mbar_init(&C.o_done, 1);
        mbar_init(&C.drain, 1);
        C.abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&C.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = C.tmem_base;
    const uint32_t tS0 = tmem;                 // S buffer 0: columns [0, 128)
    const uint32_t tO = tmem + 2 * TILE_N;     // O accumulator: columns [256, 256 + D)
    const uint64_t lim = prm.wait_limit_ns;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0 && nt > 0) {
            tma_prefetch_descriptor(&tmQ);
            tma_prefetch_descriptor(&tmK);
            tma_prefetch_descriptor(&tmV);
            mbar_arrive_expect_tx(&C.bar_q, L::Q_BYTES);
            for (int sl = 0; sl < L::SLABS; ++sl)
                tma_load_3d(sQ + sl * (MROWS * 128), &tmQ, &C.bar_q, sl * 64, qblk * BQ, bh);
        }
        int chunk = 0;  // 32 index-list entries, one per lane
        int issued = 0;
        for (int t = 0; t < nt; ++t) {
            const int s = t % NSTAGE;
            if (t >= NSTAGE) {
                const bool w = mbar_wait_bounded(&C.kv_empty[s], ((t / NSTAGE) - 1) & 1,
                                                 abort_flag, W_KV_EMPTY, lim);
                if (!__all_sync(0xFFFFFFFFu, w)) break;
            }
            const int e0 = 2 * t;
            if ((e0 & 31) == 0) {
                const int e = e0 + lane;
                chunk = (e < cnt) ? (prm.dense ? e : __ldg(idx_row + e)) : -1;
            }
            int j0 = __shfl_sync(0xFFFFFFFFu, chunk, e0 & 31);
            int j1 = __shfl_sync(0xFFFFFFFFu, chunk, (e0 + 1) & 31);
            if (e0 + 1 >= cnt) j1 = -1;
            if (j0 >= n_k || j0 < 0 || j1 >= n_k || j1 < -1) {
                if (lane == 0) record_error(SA_STATUS_DEVICE_ASSERT, 0xB000u);
                if (j0 >= n_k || j0 < 0) j0 = -1;
                if (j1 >= n_k || j1 < -1) j1 = -1;
            }
            if (lane == 0) {
                C.blk[s][0] = j0;
                C.blk[s][1] = j1;
                // An absent block is read at a row past N: TMA fills it with zeros.
                const int r0 = (j0 >= 0 ? j0 : n_k) * BK;
                const int r1 = (j1 >= 0 ? j1 : n_k) * BK;
                uint8_t* k_dst = sK + s * L::KV_BYTES;
                uint8_t* v_dst = sV + s * L::KV_BYTES;
                mbar_arrive_expect_tx(&C.k_full[s], L::KV_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl) {
                    uint8_t* base = k_dst + sl * (TILE_N * 128);
                    tma_load_3d(base, &tmK, &C.k_full[s], sl * 64, r0, bh);
                    tma_load_3d(base + BK * 128, &tmK, &C.k_full[s], sl * 64, r1, bh);
                }
                mbar_arrive_expect_tx(&C.v_full[s], L::KV_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl) {
                    uint8_t* base = v_dst + sl * (TILE_N * 128);
                    tma_load_3d(base, &tmV, &C.v_full[s], sl * 64, r0, bh);
                    tma_load_3d(base + BK * 128, &tmV, &C.v_full[s], sl * 64, r1, bh);
                }
            }
            ++issued;
        }
        // Abort path: let every copy already issued land before the CTA exits.
        if (*abort_flag && lane == 0 && nt > 0) {
            for (uint64_t t0 = globaltimer_ns();
                 !mbar_try_wait(&C.bar_q, 0) && globaltimer_ns() - t0 < lim;) {
            }
            for (int t = (issued > NSTAGE ? issued - NSTAGE : 0); t < issued; ++t) {
                const int s = t % NSTAGE;
                const uint32_t ph = (t / NSTAGE) & 1;
                for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(&C.k_full[s], ph) &&
                                                     globaltimer_ns() - t0 < lim;) {
                }
                for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(&C.v_full[s], ph) &&
                                                     globaltimer_ns() - t0 < lim;) {
                }
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0 && nt > 0) {
            constexpr uint32_t IDESC_S = make_idesc_bf16(MROWS, TILE_N, false);
            constexpr uint32_t IDESC_PV = make_idesc_bf16(MROWS, D, true);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t k_addr = smem_u32(sK);
            const uint32_t v_addr = smem_u32(sV);
            const uint32_t p_addr = smem_u32(sP);
            bool ok = mbar_wait_bounded(&C.bar_q, 0, abort_flag, W_Q, lim);
            auto issue_pv = [&](int u) -> bool {
                const int s = u % NSTAGE;
                if (!mbar_wait_bounded(&C.p_full, u & 1, abort_flag, W_P_FULL, lim)) return false;
                if (!mbar_wait_bounded(&C.v_full[s], (u / NSTAGE) & 1, abort_flag, W_V_FULL, lim))
                    return false;
                tc_fence_after();
                const uint32_t vb = v_addr + s * L::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < TILE_N / 16; ++kk) {
                    const uint64_t a = kmajor_desc(p_addr + (kk / 4) * (MROWS * 128) + (kk % 4) * 32);
                    const uint64_t b = mnmajor_desc(vb + kk * 16 * 128, TILE_N * 128);
                    umma_bf16(tO, a, b, IDESC_PV, (u > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&C.kv_empty[s]);
                umma_commit(&C.o_done);
                return true;
            };
            for (int t = 0; ok && t < nt; ++t) {
                const int s = t % NSTAGE;
                const int b = t & 1;
                if (!mbar_wait_bounded(&C.k_full[s], (t / NSTAGE) & 1, abort_flag, W_K_FULL, lim)) {
                    ok = false;
                    break;
                }
                if (t >= 2 &&
                    !mbar_wait_bounded(&C.s_free[b], ((t - 2) >> 1) & 1, abort_flag, W_S_FREE, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t kb = k_addr + s * L::KV_BYTES;
                const uint32_t dS = tS0 + b * TILE_N;
#pragma unroll
                for (int sl = 0; sl < L::SLABS; ++sl) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = kmajor_desc(q_addr + sl * (MROWS * 128) + kk * 32);
                        const uint64_t bd = kmajor_desc(kb + sl * (TILE_N * 128) + kk * 32);
                        umma_bf16(dS, a, bd, IDESC_S, (sl > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&C.s_full[b]);
                if (t >= 1 && !issue_pv(t - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) ok = issue_pv(nt - 1);
            if (!ok) {
                // Abort path: wait for every MMA issued so far before TMEM is freed.
                umma_commit(&C.drain);
                for (uint64_t t0 = globaltimer_ns();
                     !mbar_try_wait(&C.drain, 0) && globaltimer_ns() - t0 < lim;) {
                }
            }
        }
    } else {
        // ------------------------------------------- softmax and epilogue
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const int row = wq * 32 + lane;          // query row within the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const int q_tok = qblk * BQ + row;
        const bool row_valid = (row < BQ) && (q_tok < prm.N);
        const float sl2 = prm.scale_log2;
        float m_run = -INFINITY;  // running max, log2 units, as used for P
        float l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < nt; ++t) {
            const int s = t % NSTAGE;
            const int b = t & 1;
            const bool w = mbar_wait_bounded(&C.k_full[s], (t / NSTAGE) & 1, abort_flag, W_META, lim) &&
                           mbar_wait_bounded(&C.s_full[b], (t >> 1) & 1, abort_flag, W_S_FULL, lim);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int j0 = C.blk[s][0], j1 = C.blk[s][1];
            // Valid key columns of this tile: [0, v0) from block j0, [64, 64 + v1) from j1.
            const int v0 = j0 < 0 ? 0 : min(BK, prm.N - j0 * BK);
            const int v1 = j1 < 0 ? 0 : min(BK, prm.N - j1 * BK);
            float x[TILE_N];
#pragma unroll
            for (int c = 0; c < TILE_N / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tS0 + b * TILE_N + lane_off + c * 32, r);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]);
            }
            tc_fence_before();
            mbar_arrive(&C.s_free[b]);

            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < TILE_N; ++c) {
                const bool valid = (c < BK) ? (c < v0) : (c - BK < v1);
                x[c] = valid ? x[c] * sl2 : -INFINITY;
                mx = fmaxf(mx, x[c]);
            }
            float alpha = 1.f;
            if (mx > m_run + LAZY_RESCALE_LOG2) {
                alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mx);
                m_run = mx;
            }
            l_run *= alpha;
            uint32_t pk[TILE_N / 2];
            float rs = 0.f;
            if (m_run == -INFINITY) {
#pragma unroll
                for (int c = 0; c < TILE_N / 2; ++c) pk[c] = 0u;
            } else {
#pragma unroll
                for (int c = 0; c < TILE_N / 2; ++c) {
                    const float p0 = ex2_approx(x[2 * c] - m_run);
                    const float p1 = ex2_approx(x[2 * c + 1] - m_run);
                    rs += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
            }
            l_run += rs;

            // P(t-1)·V has finished: the P tile may be overwritten and O rescaled.
            if (t >= 1) {
                const bool w2 = mbar_wait_bounded(&C.o_done, (t - 1) & 1, abort_flag, W_O_DONE, lim);
                if (!__all_sync(0xFFFFFFFFu, w2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (__any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tO + lane_off + c * 32, r);
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(tO + lane_off + c * 32, r);
                    }
                }
            }
            // P tile: two 64-key slabs, each [128 rows x 128 B] with 128-byte swizzle.
#pragma unroll
            for (int c16 = 0; c16 < TILE_N / 8; ++c16) {
                const int slab = c16 / 8, chunk = c16 % 8;
                uint8_t* dst = sP + slab * (MROWS * 128) + row * 128 + ((chunk ^ (row & 7)) << 4);
                *reinterpret_cast<uint4*>(dst) =
                    make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&C.p_full);
        }

        // Epilogue: O / l, bf16, and the log-sum-exp.
        if (ok && nt > 0) {
            const bool w = mbar_wait_bounded(&C.o_done, (nt - 1) & 1, abort_flag, W_O_DONE, lim);
            ok = __all_sync(0xFFFFFFFFu, w);
            tc_fence_after();
        }
        const bool have = ok && nt > 0 && l_run > 0.f;
        const float inv_l = have ? 1.f / l_run : 0.f;
        __nv_bfloat16* out = prm.O + ((size_t)bh * prm.N + q_tok) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            if (ok && nt > 0) {
                tmem_ld32(tO + lane_off + c * 32, r);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = 0u;
            }
            if (row_valid) {
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[8 * e8 + 0]) * inv_l, __uint_as_float(r[8 * e8 + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(r[8 * e8 + 2]) * inv_l, __uint_as_float(r[8 * e8 + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(r[8 * e8 + 4]) * inv_l, __uint_as_float(r[8 * e8 + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(r[8 * e8 + 6]) * inv_l, __uint_as_float(r[8 * e8 + 7]) * inv_l);
                    *reinterpret_cast<uint4*>(out + c * 32 + 8 * e8) = v;
                }
            }
        }
        if (row_valid && prm.lse) {
            prm.lse[(size_t)bh * prm.N + q_tok] =
                have ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace fwd
}  // namespace sa
