// sa_bwd_kernels.cuh - backward pass of the block-sparse attention: dQ, dK,
// dV over the kept (query block, key block) tiles only, for sm_100a.
//
// Method: "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
// Masking and Distillation Fine-Tuning" (gist.science summary) §2B Velocity
// Distillation Fine-Tuning: the model that uses the sparse attention of §2C is
// fine-tuned, so the loss is differentiated through it. The pages print no
// formula; this is the plain derivative of the forward with the kept-block
// lists held fixed (the selection is piecewise constant in Q and K). For one
// query block with kept key tokens u, c = 1/sqrt(d), P = softmax(c Q K_u^T):
//   dV_u = P^T dO,  dP = dO V_u^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//   dQ = c dS K_u,  dK_u = c dS^T Q.
// P is recomputed from the forward's log-sum-exp, P = 2^(S c log2(e) - LSE
// log2(e)), so no row max is needed.
//
// Five launches, no atomics (the sums are deterministic):
//   bwd_rows_kernel       per query block: D and LSE log2(e) of its rows,
//                         and the block's row of a kept-block bitmap;
//   bwd_transpose_kernel  per word column of the bitmap: for each pair of
//                         adjacent key blocks (2p, 2p+1), the ascending list
//                         of the query blocks that keep either of them, with
//                         two flag bits saying which;
//   bwd_dq_kernel         query-major, like the forward: per row of kept
//                         blocks, S = Q K^T and dP = dO V^T into TMEM, dS
//                         (bf16) written back over S, dQ += dS K in TMEM;
//   bwd_dkdv_kernel       key-major: per key-block pair (128 keys), over its
//                         list of query blocks, S^T = K Q^T and dP^T = V dO^T
//                         into TMEM, P^T and dS^T (bf16) written back over
//                         them, dV += P^T dO and dK += dS^T Q in TMEM.
// The two matrix kernels share one structure: warp 8 is the TMA producer,
// warp 9 holds the tcgen05 issuer thread, warps 0-7 compute the elementwise
// step, two warpgroups taking half of a tile's columns each (a warp reads the
// TMEM lane quarter warp % 4). TMEM (512 columns):
//   dQ kernel:   S double-buffered [0,128) and [128,256), dP [256,384),
//                dQ [384,384+d): the products of tile t+1 run while the compute
//                warps turn tile t's S and dP (already in registers) into dS;
//   dK/dV kernel: S^T in two 64-column buffers [0,128), dP^T likewise
//                [128,256), dV [256,384), dK [384,512): a query block is taken in
//                halves of 64 queries, the products of one half running while the
//                compute warps form the previous half's P^T and dS^T.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"
#include "sa_attn_kernel.cuh"

namespace sa {
namespace bwd {

using attn::Desc;
using attn::desc_at;
using attn::desc_split;
using attn::kmajor_desc;
using attn::mnmajor_desc;

constexpr int BK = 64;
constexpr int TILE_N = 128;        // keys per tile of the dQ kernel; keys per work item of the dK/dV kernel
constexpr int MROWS = 128;
constexpr int NUM_THREADS = 384;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int LAUNCH_REGS = 168;
constexpr int CTRL_REGS = 56;
constexpr int COMPUTE_REGS = 224;
static_assert(128 * CTRL_REGS + 256 * COMPUTE_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;

enum WaitSite : unsigned int {
    W_Q_FULL = 0xD001, W_Q_EMPTY = 0xD002, W_CH_FULL = 0xD003, W_CH_EMPTY = 0xD004, W_S_FULL = 0xD005,
    W_P_FULL = 0xD006, W_O_FULL = 0xD007, W_ACC_FREE = 0xD008, W_KV_FULL = 0xD009, W_KV_EMPTY = 0xD00A,
    W_LOADED = 0xD00B
};

// ------------------------------------------------------------ prep kernels
// Per query block (blockIdx.x = i, blockIdx.y = bh), one thread per row r:
// lsed[(bh n_q + i) bq + r] = (LSE log2(e), D) with D = sum_c dO O, or
// (+inf, 0) past N (those rows then get P = 0). Warp 0 also writes the
// block's row of the kept-block bitmap [BH, n_q, nw] (nw = ceil(n_k / 32)
// words), recording an out-of-range or repeated index.
template <int D>
__global__ void __launch_bounds__(128)
bwd_rows_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                const float* __restrict__ lse, const int32_t* __restrict__ cnt, const int32_t* __restrict__ idx,
                float2* __restrict__ lsed, uint32_t* __restrict__ bitmap, int N, int bq, int n_q, int n_k, int nw) {
    extern __shared__ uint32_t row_bits[];
    const int i = blockIdx.x, bh = blockIdx.y;
    const int r = threadIdx.x;
    if (r < bq) {
        const int t = i * bq + r;
        float2 v = make_float2(INFINITY, 0.f);
        if (t < N) {
            const size_t off = ((size_t)bh * N + t) * D;
            const uint4* a = reinterpret_cast<const uint4*>(O + off);
            const uint4* b = reinterpret_cast<const uint4*>(dO + off);
            float acc = 0.f;
#pragma unroll 4
            for (int c = 0; c < D / 8; ++c) {
                const uint4 x = __ldg(a + c), y = __ldg(b + c);
                const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc = fmaf(__uint_as_float(xs[e] << 16), __uint_as_float(ys[e] << 16), acc);
                    acc = fmaf(__uint_as_float(xs[e] & 0xFFFF0000u), __uint_as_float(ys[e] & 0xFFFF0000u), acc);
                }
            }
            v = make_float2(lse[(size_t)bh * N + t] * LOG2E, acc);
        }
        lsed[((size_t)bh * n_q + i) * bq + r] = v;
    }
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        for (int w = lane; w < nw; w += 32) row_bits[w] = 0u;
        __syncwarp();
        const size_t row = (size_t)bh * n_q + i;
        int c = __ldg(cnt + row);
        if (c < 0 || c > n_k) {
            if (lane == 0) record_error(SA_STATUS_DEVICE_ASSERT, 0xC000u);
            c = c < 0 ? 0 : n_k;
        }
        for (int e = lane; e < c; e += 32) {
            const int j = __ldg(idx + row * n_k + e);
            if (j < 0 || j >= n_k) {
                record_error(SA_STATUS_DEVICE_ASSERT, 0xB000u);
                continue;
            }
            const uint32_t bit = 1u << (j & 31);
            if (atomicOr(&row_bits[j >> 5], bit) & bit) record_error(SA_STATUS_DEVICE_ASSERT, 0xB001u);
        }
        __syncwarp();
        for (int w = lane; w < nw; w += 32) bitmap[row * nw + w] = row_bits[w];
    }
}

// One warp per (bh, word column w): key blocks [32w, 32w + 32) = pairs
// [16w, 16w + 16). Scans the query blocks in order, 32 at a time, and
// appends (i << 2) | flags to each pair's list (flag bit 0: block 2p keeps
// i; bit 1: block 2p + 1 keeps i). ucnt[bh, p] = list length.
constexpr int TR_WARPS = 4;
__global__ void __launch_bounds__(TR_WARPS * 32)
bwd_transpose_kernel(const uint32_t* __restrict__ bitmap, int32_t* __restrict__ ucnt, int32_t* __restrict__ uidx,
                     int n_q, int nw, int n_kp) {
    const int lane = threadIdx.x & 31;
    const int w = blockIdx.x * TR_WARPS + (threadIdx.x >> 5);
    const int bh = blockIdx.y;
    if (w >= nw) return;
    int counts[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) counts[q] = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int base = 0; base < n_q; base += 32) {
        const int i = base + lane;
        const uint32_t word = i < n_q ? __ldg(bitmap + ((size_t)bh * n_q + i) * nw + w) : 0u;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int p = 16 * w + q;
            if (p >= n_kp) break;
            const uint32_t f = (word >> (2 * q)) & 3u;
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, f != 0u);
            if (f) uidx[((size_t)bh * n_kp + p) * n_q + counts[q] + __popc(bal & lt)] = (i << 2) | (int)f;
            counts[q] += __popc(bal);
        }
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const int p = 16 * w + q;
        if (lane == q && p < n_kp) ucnt[(size_t)bh * n_kp + p] = counts[q];
    }
}

// ------------------------------------------------------------ shared parts
struct Params {
    const int32_t* cnt;    // dQ kernel: [rows] kept counts;  dK/dV kernel: [items] list lengths
    const int32_t* idx;    // dQ kernel: [rows, n_k];          dK/dV kernel: [items, n_q] entries
    const float2* lsed;    // [BH * n_q * bq]: (LSE log2(e), D)
    void* out0;            // dQ kernel: dQ;  dK/dV kernel: dV   ([BH, N, d])
    void* out1;            // dK/dV kernel: dK
    int N, n_q, n_k, n_kp, items;
    int out_f32;           // 1: fp32 outputs, 0: bf16 (round to nearest even)
    float scale_log2;      // log2(e) / sqrt(d)
    float scale;           // 1 / sqrt(d)
    unsigned long long wait_limit_ns;
};

// K steps of a TS product whose A operand (bf16 pairs in TMEM) sits in two
// halves: steps [0, n/2) read a_lo + 8s, steps [n/2, n) read a_hi + 8(s - n/2).
template <int NSTEP>
__device__ __forceinline__ void umma_ts_halves(uint32_t d, uint32_t a_lo, uint32_t a_hi, const uint64_t (&b)[NSTEP],
                                               uint32_t idesc, uint32_t acc0) {
#pragma unroll
    for (int s = 0; s < NSTEP; ++s) {
        const uint32_t a = s < NSTEP / 2 ? a_lo + 8u * s : a_hi + 8u * (s - NSTEP / 2);
        umma_ts(d, a, b[s], idesc, s == 0 ? acc0 : 1u);
    }
}

// Store `n` consecutive fp32 values (registers holding bits) to a row of
// global memory as fp32 or bf16, scaled.
template <int NV>
__device__ __forceinline__ void store_row(void* base, size_t elem_off, const uint32_t (&v)[NV], float scale,
                                          bool out_f32) {
    if (out_f32) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(base) + elem_off);
#pragma unroll
        for (int e = 0; e < NV / 4; ++e)
            o[e] = make_float4(__uint_as_float(v[4 * e]) * scale, __uint_as_float(v[4 * e + 1]) * scale,
                               __uint_as_float(v[4 * e + 2]) * scale, __uint_as_float(v[4 * e + 3]) * scale);
    } else {
        uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + elem_off);
#pragma unroll
        for (int e = 0; e < NV / 8; ++e)
            o[e] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * e]) * scale, __uint_as_float(v[8 * e + 1]) * scale),
                              pack_bf16x2(__uint_as_float(v[8 * e + 2]) * scale, __uint_as_float(v[8 * e + 3]) * scale),
                              pack_bf16x2(__uint_as_float(v[8 * e + 4]) * scale, __uint_as_float(v[8 * e + 5]) * scale),
                              pack_bf16x2(__uint_as_float(v[8 * e + 6]) * scale, __uint_as_float(v[8 * e + 7]) * scale));
    }
}

template <int NV>
__device__ __forceinline__ void store_zero_row(void* base, size_t elem_off, bool out_f32) {
    if (out_f32) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(base) + elem_off);
#pragma unroll
        for (int e = 0; e < NV / 4; ++e) o[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
        uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + elem_off);
#pragma unroll
        for (int e = 0; e < NV / 8; ++e) o[e] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Elementwise step of one 32-column chunk: P = 2^(S sl2 - l2) (0 where
// !valid), dS = P (dP - Dv); packs P and dS to bf16 pairs. l2 and Dv are per
// column (dK/dV kernel) or per row (dQ kernel), given as arrays of 32.
__device__ __forceinline__ void p_ds_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], const float (&l2)[32],
                                           const float (&dv)[32], uint32_t valid_mask, float sl2,
                                           uint32_t (&pk)[16], uint32_t (&dk)[16]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint64_t y = f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])),
                                  f2_pack(sl2, sl2), f2_pack(-l2[2 * c], -l2[2 * c + 1]));
        float y0, y1;
        f2_unpack(y, y0, y1);
        float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
        if (!((valid_mask >> (2 * c)) & 1u)) p0 = 0.f;
        if (!((valid_mask >> (2 * c + 1)) & 1u)) p1 = 0.f;
        const uint64_t g = f2_mul(f2_pack(p0, p1),
                                  f2_add(f2_pack(__uint_as_float(dp[2 * c]), __uint_as_float(dp[2 * c + 1])),
                                         f2_pack(-dv[2 * c], -dv[2 * c + 1])));
        float g0, g1;
        f2_unpack(g, g0, g1);
        pk[c] = pack_bf16x2(p0, p1);
        dk[c] = pack_bf16x2(g0, g1);
    }
}

struct Ctrl {
    uint64_t q_full, q_empty;      // dQ kernel: Q and dO tiles of a row
    uint64_t ch_full[4], ch_empty[4];
    uint64_t kv_full, kv_empty;    // dK/dV kernel: K and V tiles of an item
    uint64_t qs_full[2], qs_empty[2];
    uint64_t s_full, p_full, o_full, acc_free, drain;
    uint64_t loaded;               // dQ kernel: the compute warps hold S and dP of a tile in registers
    uint64_t vch_full[2], vch_empty[2];   // dQ kernel: the V ring (the K ring uses ch_full/ch_empty)
    uint64_t s2_full[2], p2_full[2];      // dK/dV kernel: per TMEM buffer of a 64-query unit
    uint32_t tmem_base;
    int abort_flag;
};

// ------------------------------------------------------------ dQ kernel
template <int D, int BQ>
struct DQLayout {
    static constexpr int SLABS = D / 64;
    static constexpr int TILE_BYTES = MROWS * D * 2;   // Q, dO, and each K or V tile (128 rows)
    // Separate rings: a V tile is free once its dP product is done, a K tile
    // only after its dQ product; three K slots let K(t+1) land while K(t-1)
    // and K(t) are still in use.
    static constexpr int NKS = 3, NVS = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = TILE_BYTES;
    static constexpr int OFF_K = 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NKS * TILE_BYTES;
    static constexpr int OFF_CTRL = OFF_V + NVS * TILE_BYTES;
    static constexpr int DYN_BYTES = OFF_CTRL + 512 + 1024;
    static_assert(DYN_BYTES <= 232448, "shared memory budget");
};

template <int D, int BQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO, const Params prm) {
    using L = DQLayout<D, BQ>;
    constexpr int NKS = L::NKS, NVS = L::NVS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl& C = *reinterpret_cast<Ctrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_k = prm.n_k, rows = prm.items;
    const uint64_t lim = prm.wait_limit_ns;

    if (threadIdx.x == 0) {
        mbar_init(&C.q_full, 1);
        mbar_init(&C.q_empty, 1);
        for (int c = 0; c < NKS; ++c) {
            mbar_init(&C.ch_full[c], 1);
            mbar_init(&C.ch_empty[c], 1);
        }
        for (int c = 0; c < NVS; ++c) {
            mbar_init(&C.vch_full[c], 1);
            mbar_init(&C.vch_empty[c], 1);
        }
        mbar_init(&C.s_full, 1);
        mbar_init(&C.p_full, 8);
        mbar_init(&C.o_full, 1);
        mbar_init(&C.acc_free, 8);
        mbar_init(&C.drain, 1);
        mbar_init(&C.loaded, 8);
        C.abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(&C.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = C.tmem_base;
    auto count_of = [&](int r) -> int {
        int c = __ldg(prm.cnt + r);
        return (c < 0 || c > n_k) ? (c < 0 ? 0 : n_k) : c;   // a bad count was recorded by bwd_rows_kernel
    };
    auto entry_of = [&](int r, int c, int e) -> int {
        if (e >= c) return -1;
        const int j = __ldg(prm.idx + (size_t)r * n_k + e);
        return (j >= 0 && j < n_k) ? j : -1;   // out of range: skipped (recorded by bwd_rows_kernel)
    };

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTRL_REGS));
        if (warp == PRODUCER_WARP) {
            if (lane == 0) {
                tma_prefetch_descriptor(&tmQ);
                tma_prefetch_descriptor(&tmK);
                tma_prefetch_descriptor(&tmV);
                tma_prefetch_descriptor(&tmdO);
            }
            int g = 0, kq = 0;     // tiles loaded so far (both rings advance once per tile)
            int gk = 0, gv = 0;    // K and V copies issued (for the abort drain)
            bool ok = true;
            for (int r = blockIdx.x; ok && r < rows; r += gridDim.x) {
                const int cnt = count_of(r);
                const int nt = (cnt + 1) / 2;
                if (nt == 0) continue;
                const int bh = r / prm.n_q, qb = r % prm.n_q;
                if (kq > 0 && !wait_warp(&C.q_empty, (kq - 1) & 1, abort_flag, W_Q_EMPTY, lim)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&C.q_full, 2 * L::TILE_BYTES);
                    for (int sl = 0; sl < L::SLABS; ++sl) {
                        tma_load_3d(smem + L::OFF_Q + sl * (MROWS * 128), &tmQ, &C.q_full, sl * 64, qb * BQ, bh);
                        tma_load_3d(smem + L::OFF_DO + sl * (MROWS * 128), &tmdO, &C.q_full, sl * 64, qb * BQ, bh);
                    }
                }
                ++kq;
                int window = -1;
                for (int t = 0; t < nt; ++t, ++g) {
                    const int e0 = 2 * t;
                    if ((e0 & 31) == 0) window = entry_of(r, cnt, e0 + lane);
                    int j0 = __shfl_sync(0xFFFFFFFFu, window, e0 & 31);
                    int j1 = __shfl_sync(0xFFFFFFFFu, window, (e0 + 1) & 31);
                    // An absent (or skipped) block is read at a row past N: zeros.
                    const int r0 = (j0 >= 0 ? j0 : n_k) * BK;
                    const int r1 = (j1 >= 0 ? j1 : n_k) * BK;
                    const int ck = g % NKS, cv = g % NVS;
                    if (g >= NKS && !wait_warp(&C.ch_empty[ck], ((g / NKS) - 1) & 1, abort_flag, W_CH_EMPTY, lim)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        uint8_t* dst = smem + L::OFF_K + ck * L::TILE_BYTES;
                        mbar_arrive_expect_tx(&C.ch_full[ck], L::TILE_BYTES);
                        for (int sl = 0; sl < L::SLABS; ++sl) {
                            tma_load_3d(dst + sl * (TILE_N * 128), &tmK, &C.ch_full[ck], sl * 64, r0, bh);
                            tma_load_3d(dst + sl * (TILE_N * 128) + BK * 128, &tmK, &C.ch_full[ck], sl * 64, r1, bh);
                        }
                    }
                    gk = g + 1;
                    if (g >= NVS && !wait_warp(&C.vch_empty[cv], ((g / NVS) - 1) & 1, abort_flag, W_CH_EMPTY, lim)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        uint8_t* dst = smem + L::OFF_V + cv * L::TILE_BYTES;
                        mbar_arrive_expect_tx(&C.vch_full[cv], L::TILE_BYTES);
                        for (int sl = 0; sl < L::SLABS; ++sl) {
                            tma_load_3d(dst + sl * (TILE_N * 128), &tmV, &C.vch_full[cv], sl * 64, r0, bh);
                            tma_load_3d(dst + sl * (TILE_N * 128) + BK * 128, &tmV, &C.vch_full[cv], sl * 64, r1, bh);
                        }
                    }
                    gv = g + 1;
                }
            }
            if (*abort_flag && lane == 0) {
                // Every copy issued must land before the CTA's shared memory is released.
                if (kq > 0) drain_wait(&C.q_full, (kq - 1) & 1, lim);
                for (int gg = (gk > NKS ? gk - NKS : 0); gg < gk; ++gg) drain_wait(&C.ch_full[gg % NKS], (gg / NKS) & 1, lim);
                for (int gg = (gv > NVS ? gv - NVS : 0); gg < gv; ++gg) drain_wait(&C.vch_full[gg % NVS], (gg / NVS) & 1, lim);
            }
        } else if (warp == MMA_WARP && lane == 0) {
            constexpr uint32_t IDESC_S = make_idesc_bf16(MROWS, TILE_N, false);
            constexpr uint32_t IDESC_DQ = make_idesc_bf16(MROWS, D, true);
            const Desc q_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_Q)));
            const Desc do_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_DO)));
            const Desc k_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_K)));
            const Desc v_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_V)));
            const Desc k_mn = desc_split(mnmajor_desc(smem_u32(smem + L::OFF_K), TILE_N * 128));
            // S is double-buffered: the products of tile g + 1 go out as soon as the
            // compute warps have read tile g's S and dP into registers.
            // S buffer b at tmem + 128 b.
            const uint32_t tdP = tmem + 256, tdQ = tmem + 384;
            int g = 0, kq = 0, rown = 0;
            bool ok = true;
            // S or dP (into d) = A (128 rows, K-major) times B^T (a ring slot, K-major).
            auto issue_sk = [&](uint32_t d, Desc a, Desc b, int slot) {
                const uint32_t coff = (uint32_t)(slot * L::TILE_BYTES) >> 4;
#pragma unroll
                for (int sl = 0; sl < L::SLABS; ++sl)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t o = (sl * (MROWS * 128) + kk * 32) >> 4;
                        umma_ss(d, desc_at(a, o), desc_at(b, coff + o), IDESC_S, (sl | kk) ? 1u : 0u);
                    }
            };
            // The products of tile gt (K in ring slot gt % NKS, V in gt % NVS), into S buffer gt & 1.
            auto issue_products = [&](int gt) -> bool {
                const int ck = gt % NKS, cv = gt % NVS;
                if (!mbar_wait_spin(&C.ch_full[ck], (gt / NKS) & 1, abort_flag, W_CH_FULL, lim) ||
                    !mbar_wait_spin(&C.vch_full[cv], (gt / NVS) & 1, abort_flag, W_CH_FULL, lim))
                    return false;
                tc_fence_after();
                issue_sk(tmem + 128u * (gt & 1), q_desc, k_desc, ck);
                issue_sk(tdP, do_desc, v_desc, cv);
                umma_commit(&C.s_full);
                umma_commit(&C.vch_empty[cv]);          // V is no longer needed
                return true;
            };
            for (int r = blockIdx.x; ok && r < rows; r += gridDim.x) {
                const int nt = (count_of(r) + 1) / 2;
                if (nt == 0) continue;
                if (!mbar_wait_spin(&C.q_full, kq & 1, abort_flag, W_Q_FULL, lim)) { ok = false; break; }
                ++kq;
                // The first tile's dP overwrites the previous tile's, which the
                // compute warps must have read.
                if (g > 0 && !mbar_wait_spin(&C.loaded, (g - 1) & 1, abort_flag, W_LOADED, lim)) { ok = false; break; }
                if (!issue_products(g)) { ok = false; break; }
                if (nt == 1) umma_commit(&C.q_empty);
                for (int t = 0; t < nt; ++t) {
                    if (t + 1 < nt) {
                        if (!mbar_wait_spin(&C.loaded, g & 1, abort_flag, W_LOADED, lim) ||
                            !issue_products(g + 1)) {
                            ok = false;
                            break;
                        }
                        if (t + 2 == nt) umma_commit(&C.q_empty);
                    }
                    if (!mbar_wait_spin(&C.p_full, g & 1, abort_flag, W_P_FULL, lim)) { ok = false; break; }
                    if (t == 0 && rown > 0 && !mbar_wait_spin(&C.acc_free, (rown - 1) & 1, abort_flag, W_ACC_FREE, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int ck = g % NKS;
                    uint64_t bk[TILE_N / 16];
                    const uint32_t coff = (uint32_t)(ck * L::TILE_BYTES) >> 4;
#pragma unroll
                    for (int kk = 0; kk < TILE_N / 16; ++kk) bk[kk] = desc_at(k_mn, coff + ((kk * 16 * 128) >> 4));
                    const uint32_t tSg = tmem + 128u * (g & 1);
                    umma_ts_halves<TILE_N / 16>(tdQ, tSg, tSg + 64, bk, IDESC_DQ, t > 0 ? 1u : 0u);
                    umma_commit(&C.ch_empty[ck]);          // K is no longer needed
                    if (t + 1 == nt) umma_commit(&C.o_full);
                    ++g;
                }
                ++rown;
            }
            if (!ok) {
                umma_commit(&C.drain);
                drain_wait(&C.drain, 0, lim);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(COMPUTE_REGS));
        const int wg = warp / 4;                 // column half of a tile
        const int wq = warp & 3;                 // TMEM lane quarter
        const int row = wq * 32 + lane;          // query row within the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        // S buffer b at tmem + lane_off + 128 b.
        const uint32_t tdP = tmem + 256 + lane_off, tdQ = tmem + 384 + lane_off;
        const float sl2 = prm.scale_log2;
        const bool f32 = prm.out_f32 != 0;
        int g = 0, rown = 0;
        bool ok = true;
        for (int r = blockIdx.x; ok && r < rows; r += gridDim.x) {
            const int cnt = count_of(r);
            const int nt = (cnt + 1) / 2;
            const int bh = r / prm.n_q, qb = r % prm.n_q;
            const int q_tok = qb * BQ + row;
            const bool row_valid = row < BQ && q_tok < prm.N;
            const size_t out_off = ((size_t)bh * prm.N + q_tok) * D + wg * (D / 2);
            if (nt == 0) {
                if (row_valid) store_zero_row<D / 2>(prm.out0, out_off, f32);
                continue;
            }
            float2 ld = make_float2(INFINITY, 0.f);
            if (row_valid) ld = prm.lsed[((size_t)bh * prm.n_q + qb) * BQ + row];
            float l2[32], dv[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                l2[c] = ld.x;
                dv[c] = ld.y;
            }
            int window = -1;
            for (int t = 0; t < nt; ++t) {
                const int e0 = 2 * t;
                if ((e0 & 31) == 0) window = entry_of(r, cnt, e0 + lane);
                // This warpgroup's 64 columns are the keys of one block of the tile.
                const int jb = __shfl_sync(0xFFFFFFFFu, window, (e0 + wg) & 31);
                const int j = (e0 + wg < cnt) ? jb : -1;
                const int nvalid = j < 0 ? 0 : min(BK, prm.N - j * BK);
                if (!wait_warp(&C.s_full, g & 1, abort_flag, W_S_FULL, lim)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tS = tmem + lane_off + 128u * (g & 1);
                uint32_t s[64], dp[64];
                tmem_ld64(tS + wg * 64, s);
                tmem_ld64(tdP + wg * 64, dp);
                // S and dP are in registers: the next tile's products may overwrite dP.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&C.loaded);
#pragma unroll
                for (int h = 0; h < 2; ++h) {   // two chunks of 32 keys
                    const int nv = nvalid - h * 32;
                    const uint32_t vm = nv >= 32 ? 0xFFFFFFFFu : (nv <= 0 ? 0u : ((1u << nv) - 1u));
                    uint32_t pk[16], dk[16];
                    p_ds_chunk(*reinterpret_cast<const uint32_t(*)[32]>(s + 32 * h),
                               *reinterpret_cast<const uint32_t(*)[32]>(dp + 32 * h), l2, dv, vm, sl2, pk, dk);
                    // dS goes over this warpgroup's own S columns (already read).
                    tmem_st16_nowait(tS + wg * 64 + h * 16, dk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&C.p_full);
                ++g;
            }
            if (!ok) break;
            if (!wait_warp(&C.o_full, rown & 1, abort_flag, W_O_FULL, lim)) { ok = false; break; }
            tc_fence_after();
            uint32_t o[D / 2];
            if constexpr (D == 128) tmem_ld64(tdQ + wg * 64, o); else tmem_ld32(tdQ + wg * 32, o);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&C.acc_free);
            ++rown;
            if (row_valid) store_row<D / 2>(prm.out0, out_off, o, prm.scale, f32);
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------ dK/dV kernel
template <int D, int BQ>
struct KVLayout {
    static constexpr int SLABS = D / 64;
    static constexpr int KV_BYTES = TILE_N * D * 2;    // K or V of a key-block pair
    static constexpr int QT_BYTES = BQ * D * 2;        // Q or dO of a query block
    static constexpr int LSED_BYTES = BQ * 8;
    static constexpr int NST = 2;                      // query-block stages
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = KV_BYTES;
    static constexpr int OFF_ST = 2 * KV_BYTES;        // stage s: Q at OFF_ST + s*2*QT, dO after it
    static constexpr int OFF_LSED = OFF_ST + NST * 2 * QT_BYTES;
    static constexpr int OFF_CTRL = OFF_LSED + NST * LSED_BYTES;
    static constexpr int DYN_BYTES = OFF_CTRL + 512 + 1024;
    static_assert(DYN_BYTES <= 232448, "shared memory budget");
    static_assert(QT_BYTES % 1024 == 0, "swizzled tiles stay 1024-byte aligned");
};

template <int D, int BQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO, const Params prm) {
    using L = KVLayout<D, BQ>;
    constexpr int NST = L::NST;
    constexpr int NH = BQ / 64;              // 64-query units per query block
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl& C = *reinterpret_cast<Ctrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_q = prm.n_q, items = prm.items;
    const uint64_t lim = prm.wait_limit_ns;

    if (threadIdx.x == 0) {
        mbar_init(&C.kv_full, 1);
        mbar_init(&C.kv_empty, 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&C.qs_full[s], 1);
            mbar_init(&C.qs_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&C.s2_full[b], 1);
            mbar_init(&C.p2_full[b], 8);
        }
        mbar_init(&C.o_full, 1);
        mbar_init(&C.acc_free, 8);
        mbar_init(&C.drain, 1);
        C.abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(&C.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = C.tmem_base;
    auto count_of = [&](int it) -> int {
        const int c = __ldg(prm.cnt + it);
        return (c < 0 || c > n_q) ? 0 : c;   // written by bwd_transpose_kernel: always in range
    };
    auto entry_of = [&](int it, int c, int e) -> int {
        return e < c ? __ldg(prm.idx + (size_t)it * n_q + e) : 0;
    };

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTRL_REGS));
        if (warp == PRODUCER_WARP) {
            if (lane == 0) {
                tma_prefetch_descriptor(&tmQ);
                tma_prefetch_descriptor(&tmK);
                tma_prefetch_descriptor(&tmV);
                tma_prefetch_descriptor(&tmdO);
            }
            int itn = 0, es = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
                const int cnt = count_of(it);
                if (cnt == 0) continue;
                const int bh = it / prm.n_kp, pr = it % prm.n_kp;
                if (itn > 0 && !wait_warp(&C.kv_empty, (itn - 1) & 1, abort_flag, W_KV_EMPTY, lim)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&C.kv_full, 2 * L::KV_BYTES);
                    for (int sl = 0; sl < L::SLABS; ++sl)
                        for (int hb = 0; hb < 2; ++hb) {
                            const int off = sl * (TILE_N * 128) + hb * (BK * 128);
                            const int row0 = (2 * pr + hb) * BK;   // past N: zeros
                            tma_load_3d(smem + L::OFF_K + off, &tmK, &C.kv_full, sl * 64, row0, bh);
                            tma_load_3d(smem + L::OFF_V + off, &tmV, &C.kv_full, sl * 64, row0, bh);
                        }
                }
                ++itn;
                int window = 0;
                for (int e = 0; e < cnt; ++e) {
                    if ((e & 31) == 0) window = entry_of(it, cnt, e + lane);
                    const int qb = __shfl_sync(0xFFFFFFFFu, window, e & 31) >> 2;
                    const int st = es % NST;
                    if (es >= NST && !wait_warp(&C.qs_empty[st], ((es / NST) - 1) & 1, abort_flag, W_Q_EMPTY, lim)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        uint8_t* sq = smem + L::OFF_ST + st * 2 * L::QT_BYTES;
                        mbar_arrive_expect_tx(&C.qs_full[st], 2 * L::QT_BYTES + L::LSED_BYTES);
                        for (int sl = 0; sl < L::SLABS; ++sl) {
                            tma_load_3d(sq + sl * (BQ * 128), &tmQ, &C.qs_full[st], sl * 64, qb * BQ, bh);
                            tma_load_3d(sq + L::QT_BYTES + sl * (BQ * 128), &tmdO, &C.qs_full[st], sl * 64, qb * BQ, bh);
                        }
                        bulk_load_1d(smem + L::OFF_LSED + st * L::LSED_BYTES,
                                     prm.lsed + ((size_t)bh * n_q + qb) * BQ, L::LSED_BYTES, &C.qs_full[st]);
                    }
                    ++es;
                }
            }
            if (*abort_flag && lane == 0) {
                if (itn > 0) drain_wait(&C.kv_full, (itn - 1) & 1, lim);
                for (int ee = (es > NST ? es - NST : 0); ee < es; ++ee) drain_wait(&C.qs_full[ee % NST], (ee / NST) & 1, lim);
            }
        } else if (warp == MMA_WARP && lane == 0) {
            // Query blocks are processed in halves of 64 queries ("units"); S^T
            // and dP^T of a unit go to buffer unit & 1 (64 columns each), so the
            // products of unit u+1 run while the compute warps form unit u's
            // weights, and dV, dK of unit u follow.
            constexpr uint32_t IDESC_ST = make_idesc_bf16(MROWS, 64, false);
            constexpr uint32_t IDESC_G = make_idesc_bf16(MROWS, D, true);
            const Desc k_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_K)));
            const Desc v_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_V)));
            const Desc st_desc = desc_split(kmajor_desc(smem_u32(smem + L::OFF_ST)));
            const Desc st_mn = desc_split(mnmajor_desc(smem_u32(smem + L::OFF_ST), BQ * 128));
            const uint32_t tdV = tmem + 256, tdK = tmem + 384;
            int itn = 0, es = 0, gu = 0;
            bool ok = true;
            // d = A (K or V pair tile, 128 rows) times B^T (64 rows of Q or dO at b_off16).
            auto issue_t = [&](uint32_t d, Desc a, uint32_t b_off16) {
#pragma unroll
                for (int sl = 0; sl < L::SLABS; ++sl)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_ss(d, desc_at(a, (sl * (TILE_N * 128) + kk * 32) >> 4),
                                desc_at(st_desc, b_off16 + ((sl * (BQ * 128) + kk * 32) >> 4)), IDESC_ST,
                                (sl | kk) ? 1u : 0u);
            };
            // Offsets (16-byte units) of unit v's Q and dO rows in the stage ring.
            auto q_off_of = [&](int e_glob, int hf) -> uint32_t {
                return (uint32_t)((e_glob % NST) * 2 * L::QT_BYTES + hf * 64 * 128) >> 4;
            };
            // dV, dK of the unit gu_u (entry e_glob, half hf); first = it overwrites.
            auto issue_grad = [&](int gu_u, int e_glob, int hf, bool first) {
                const uint32_t qo = q_off_of(e_glob, hf);
                const uint32_t doo = qo + ((uint32_t)L::QT_BYTES >> 4);
                uint64_t bq_do[4], bq_q[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    bq_q[kk] = desc_at(st_mn, qo + ((kk * 16 * 128) >> 4));
                    bq_do[kk] = desc_at(st_mn, doo + ((kk * 16 * 128) >> 4));
                }
                const uint32_t tSu = tmem + 64u * (gu_u & 1), tdPu = tmem + 128 + 64u * (gu_u & 1);
                umma_ts_halves<4>(tdV, tSu, tSu + 32, bq_do, IDESC_G, first ? 0u : 1u);
                umma_ts_halves<4>(tdK, tdPu, tdPu + 32, bq_q, IDESC_G, first ? 0u : 1u);
                if (hf == NH - 1) umma_commit(&C.qs_empty[e_glob % NST]);
            };
            for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
                const int cnt = count_of(it);
                if (cnt == 0) continue;
                if (!mbar_wait_spin(&C.kv_full, itn & 1, abort_flag, W_KV_FULL, lim)) { ok = false; break; }
                const int nu = cnt * NH;
                for (int v = 0; v < nu; ++v, ++gu) {
                    const int e_glob = es + v / NH, hf = v % NH;
                    if (hf == 0 &&
                        !mbar_wait_spin(&C.qs_full[e_glob % NST], (e_glob / NST) & 1, abort_flag, W_Q_FULL, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t qo = q_off_of(e_glob, hf);
                    issue_t(tmem + 64u * (gu & 1), k_desc, qo);
                    issue_t(tmem + 128 + 64u * (gu & 1), v_desc, qo + ((uint32_t)L::QT_BYTES >> 4));
                    umma_commit(&C.s2_full[gu & 1]);
                    if (v >= 1) {
                        const int pu = gu - 1, pe = es + (v - 1) / NH, ph = (v - 1) % NH;
                        if (!mbar_wait_spin(&C.p2_full[pu & 1], (pu >> 1) & 1, abort_flag, W_P_FULL, lim) ||
                            (v == 1 && itn > 0 &&
                             !mbar_wait_spin(&C.acc_free, (itn - 1) & 1, abort_flag, W_ACC_FREE, lim))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_grad(pu, pe, ph, v == 1);
                    }
                }
                if (!ok) break;
                // The item's last unit.
                {
                    const int pu = gu - 1, pe = es + (nu - 1) / NH, ph = (nu - 1) % NH;
                    if (!mbar_wait_spin(&C.p2_full[pu & 1], (pu >> 1) & 1, abort_flag, W_P_FULL, lim) ||
                        (nu == 1 && itn > 0 && !mbar_wait_spin(&C.acc_free, (itn - 1) & 1, abort_flag, W_ACC_FREE, lim))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_grad(pu, pe, ph, nu == 1);
                }
                es += cnt;
                umma_commit(&C.o_full);
                umma_commit(&C.kv_empty);
                ++itn;
            }
            if (!ok) {
                umma_commit(&C.drain);
                drain_wait(&C.drain, 0, lim);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(COMPUTE_REGS));
        const int wg = warp / 4;                 // 32 of a unit's 64 query columns each
        const int wq = warp & 3;
        const int row = wq * 32 + lane;          // key within the pair tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tdV = tmem + 256 + lane_off, tdK = tmem + 384 + lane_off;
        const float sl2 = prm.scale_log2;
        const bool f32 = prm.out_f32 != 0;
        int itn = 0, es = 0, gu = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
            const int cnt = count_of(it);
            const int bh = it / prm.n_kp, pr = it % prm.n_kp;
            const int key = pr * TILE_N + row;
            const bool key_valid = key < prm.N;
            const int half = row >> 6;           // which block of the pair this key is in
            void* out = wg == 0 ? prm.out0 : prm.out1;   // warpgroup 0 writes dV, 1 writes dK
            const size_t out_off = ((size_t)bh * prm.N + key) * D;
            if (cnt == 0) {
                if (key_valid) store_zero_row<D>(out, out_off, f32);
                continue;
            }
            int window = 0;
            for (int e = 0; e < cnt; ++e) {
                if ((e & 31) == 0) window = entry_of(it, cnt, e + lane);
                const int ent = __shfl_sync(0xFFFFFFFFu, window, e & 31);
                const bool kept = key_valid && ((ent >> half) & 1);
                const int eg = es + e, st = eg % NST;
                // The stage's LSE and D values are read from shared memory: wait for its copy too.
                if (!wait_warp(&C.qs_full[st], (eg / NST) & 1, abort_flag, W_Q_FULL, lim)) { ok = false; break; }
                const float2* lsed = reinterpret_cast<const float2*>(smem + L::OFF_LSED + st * L::LSED_BYTES);
                for (int hf = 0; hf < NH; ++hf, ++gu) {
                    const int b = gu & 1;
                    if (!wait_warp(&C.s2_full[b], (gu >> 1) & 1, abort_flag, W_S_FULL, lim)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t tS = tmem + lane_off + 64u * b, tdP = tmem + 128 + lane_off + 64u * b;
                    uint32_t s[32], dp[32];
                    tmem_ld32(tS + wg * 32, s);
                    tmem_ld32(tdP + wg * 32, dp);
                    float l2[32], dv[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float2 v = lsed[hf * 64 + wg * 32 + c];
                        l2[c] = v.x;
                        dv[c] = v.y;
                    }
                    uint32_t pk[16], dk[16];
                    p_ds_chunk(s, dp, l2, dv, kept ? 0xFFFFFFFFu : 0u, sl2, pk, dk);
                    // Over this warpgroup's own S^T and dP^T columns (already read).
                    tmem_st16_nowait(tS + wg * 32, pk);
                    tmem_st16_nowait(tdP + wg * 32, dk);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&C.p2_full[b]);
                }
                if (!ok) break;
            }
            es += cnt;
            if (!ok) break;
            if (!wait_warp(&C.o_full, itn & 1, abort_flag, W_O_FULL, lim)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tacc = wg == 0 ? tdV : tdK;
            const float sc = wg == 0 ? 1.f : prm.scale;
            uint32_t o[D / 2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if constexpr (D == 128) tmem_ld64(tacc + h * 64, o); else tmem_ld32(tacc + h * 32, o);
                if (h == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&C.acc_free);
                }
                if (key_valid) store_row<D / 2>(out, out_off + h * (D / 2), o, sc, f32);
            }
            ++itn;
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace bwd
}  // namespace sa
