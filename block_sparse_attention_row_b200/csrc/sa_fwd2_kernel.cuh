// sa_fwd2_kernel.cuh - step 4 of the path: block-sparse FlashAttention-style
// forward over the kept (query block, key block) tiles only, for sm_100a.
//
// Method: "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
// Masking and Distillation Fine-Tuning" (gist.science summary) §2C Efficient
// Kernel Implementation: the tensors are split into tiles, the hybrid mask is
// applied per block, and the matmuls and softmax of masked tiles are skipped.
// Here a masked tile is never loaded, multiplied or exponentiated: each query
// block walks only its own kept-block list.
//
// One CTA serves two query-block rows ("slots") at once so that the tensor
// cores always have one slot's matmuls to run while the other slot's softmax
// is computed. 384 threads in four roles:
//   warp 8      TMA producer: each slot's Q tile once, then K and V chunks
//               (two kept key blocks = 128 keys per chunk) gathered by the
//               slots' index lists into a ring of 32 KB chunks, in a fixed
//               interleaved order both the producer and the MMA issuer walk;
//   warp 9      tcgen05 issuer (one thread): S_s = Q_s K^T into TMEM, then
//               O_s += P_s V with P_s read from TMEM where the softmax wrote it
//               over S_s (the next S_s is issued after that product, and the
//               tensor pipe executes one thread's MMAs in order);
//   warps 0-3   softmax of slot 0, warps 4-7 softmax of slot 1: one query row
//               per thread (one TMEM lane), base-2 online softmax with a lazy
//               rescale of O (only when the running max grows by more than
//               2^8); a quarter of the exponentials run as a polynomial on the
//               FMA pipe to offload the MUFU unit; then the epilogue.
//   warps 10-11 idle. The control warpgroup (8-11) hands most of its
//               registers to the two softmax warpgroups (setmaxnreg).
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d),
// O_1 [384,384+d); P_s (bf16 pairs) overwrites the first 64 columns of S_s.
// Tensor-core shapes: S tile M=128 x N=128 x K=d (A, B from shared memory);
// PV tile M=128 x N=d x K=128 (A from TMEM, B = V from shared memory).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"

namespace sa {
namespace fwd2 {

constexpr int BK = 64;           // key block (tokens)
constexpr int TILE_N = 128;      // keys per chunk: two kept key blocks
constexpr int MROWS = 128;       // query rows per MMA tile
constexpr int NSLOT = 2;         // query-block rows per CTA
constexpr int NUM_THREADS = 384;   // softmax warpgroups 0-1, control warpgroup 2
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
// Register split (setmaxnreg): the kernel launches with LAUNCH_REGS per thread
// (384 x 168 = 64512 registers); the control warpgroup gives back down to
// CTRL_REGS and the two softmax warpgroups take the rest:
// 128 x 40 + 256 x 232 = 64512.
constexpr int LAUNCH_REGS = 168;
constexpr int CTRL_REGS = 40;
constexpr int SOFTMAX_REGS = 232;
static_assert(128 * CTRL_REGS + 256 * SOFTMAX_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;
// One column pair in EXP_POLY_EVERY takes its exponentials on the FMA pipe
// (exp2_poly) instead of the MUFU unit; 0 keeps every exponential on MUFU.
// Measured on B200: the MUFU unit is not the limit of this kernel, and the
// polynomial's extra instructions lengthen the softmax, so it is off.
constexpr int EXP_POLY_EVERY = 0;
constexpr int MAX_CHUNKS = 10;

// Where a bounded wait gave up (reported in the device error record).
enum WaitSite : unsigned int {
    W_CH_EMPTY = 0xE001, W_Q = 0xE002, W_CH_FULL = 0xE003, W_P_FULL = 0xE004,
    W_S_FULL = 0xE005, W_O_DONE = 0xE006
};

template <int D>
struct Layout2 {
    static constexpr int SLABS = D / 64;                 // 64-channel (128-byte) slabs
    static constexpr int Q_BYTES = MROWS * D * 2;        // per slot
    static constexpr int CH_BYTES = TILE_N * D * 2;      // one K or V chunk
    static constexpr int NCHUNK = (D == 128) ? 5 : 10;   // ring depth
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_CH = NSLOT * Q_BYTES;
    static constexpr int OFF_CTRL = OFF_CH + NCHUNK * CH_BYTES;
    static constexpr int CTRL_BYTES = 512;
    static constexpr int DYN_BYTES = OFF_CTRL + CTRL_BYTES + 1024;
    static_assert(NCHUNK <= MAX_CHUNKS, "chunk ring too deep");
    static_assert(DYN_BYTES <= 232448, "shared memory budget");
    static_assert(DYN_BYTES > 116 * 1024, "one CTA per SM (TMEM is allocated whole)");
};

struct Ctrl2 {
    uint64_t q_full[NSLOT];
    uint64_t ch_full[MAX_CHUNKS];
    uint64_t ch_empty[MAX_CHUNKS];
    uint64_t s_full[NSLOT];
    uint64_t p_full[NSLOT];
    uint64_t o_done[NSLOT];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct Fwd2Params {
    const int32_t* cnt;  // [BH * n_q]
    const int32_t* idx;  // [BH * n_q, n_k]
    void* O;             // [BH, N, D], bf16 or fp32 (out_f32)
    float* lse;          // [BH, N] or null
    int N, n_q, n_k, rows;
    int dense;           // 1: every key block, no index list
    int out_f32;         // 1: O is fp32, 0: bf16 (round to nearest even)
    float scale_log2;    // log2(e) / sqrt(d)
    unsigned long long wait_limit_ns;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
    return make_sdesc_sw128(addr, 16u, 1024u);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr, uint32_t slab_bytes) {
    return make_sdesc_sw128(addr, slab_bytes, 1024u);
}

// 2^x on the FMA pipe for x <= 8 (Cody-Waite range reduction x = n + f with
// n = round(x), f in [-1/2, 1/2], and a degree-3 Remez polynomial for 2^f of
// relative error 7.5e-5; coefficients from csrc/gen_exp2_poly.py). Inputs
// below -125 are clamped (their weight is far below bf16 resolution); -inf
// gives exactly 0.
__device__ __forceinline__ float exp2_poly(float x) {
    const float xc = fmaxf(x, -125.0f);
    const float t = xc + 12582912.0f;            // 1.5 * 2^23: round to an integer
    const float f = xc - (t - 12582912.0f);      // f in [-1/2, 1/2]
    float pf = fmaf(5.517166853e-02f, f, 2.426111251e-01f);
    pf = fmaf(pf, f, 6.932609677e-01f);
    pf = fmaf(pf, f, 9.999280572e-01f);
    // bits(t) << 23 equals round(x) << 23: the low 9 bits of bits(1.5*2^23) are zero.
    const float r = __uint_as_float(__float_as_uint(pf) + (__float_as_uint(t) << 23));
    return (x == -INFINITY) ? 0.f : r;
}

// exp2_poly on a pair of fp32 values held as one .f32x2 register, with the
// range reduction and the polynomial in paired arithmetic.
__device__ __forceinline__ void exp2_poly_pair(uint64_t y, float& r0, float& r1) {
    float y0, y1;
    f2_unpack(y, y0, y1);
    const uint64_t a = f2_pack(fmaxf(y0, -125.0f), fmaxf(y1, -125.0f));
    const uint64_t t = f2_add(a, f2_pack(12582912.0f, 12582912.0f));
    const uint64_t u = f2_add(t, f2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f2_fma(u, f2_pack(-1.0f, -1.0f), a);
    uint64_t q = f2_fma(f2_pack(5.517166853e-02f, 5.517166853e-02f), f,
                        f2_pack(2.426111251e-01f, 2.426111251e-01f));
    q = f2_fma(q, f, f2_pack(6.932609677e-01f, 6.932609677e-01f));
    q = f2_fma(q, f, f2_pack(9.999280572e-01f, 9.999280572e-01f));
    float q0, q1, t0, t1;
    f2_unpack(q, q0, q1);
    f2_unpack(t, t0, t1);
    r0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
    r1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
    r0 = (y0 == -INFINITY) ? 0.f : r0;
    r1 = (y1 == -INFINITY) ? 0.f : r1;
}

// The MMA issuer keeps each shared-memory descriptor as a (low, high) word
// pair: moving the start address by a byte offset adds offset >> 4 to the
// low word (offsets stay below 2^18 bytes, so the 14-bit field never
// carries), which keeps the instructions between two MMAs to a minimum.
struct Desc {
    uint32_t lo, hi;
};
__device__ __forceinline__ Desc desc_split(uint64_t d) {
    return {static_cast<uint32_t>(d), static_cast<uint32_t>(d >> 32)};
}

// D[tmem] (+)= A[smem] * B[smem], bf16, fp32 accumulate; descriptors as word pairs.
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, Desc a, uint32_t a_off16, Desc b,
                                        uint32_t b_off16, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"
        "mov.b64 ad, {%1, %2};\n\t"
        "mov.b64 bd, {%3, %4};\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a.lo + a_off16), "r"(a.hi), "r"(b.lo + b_off16), "r"(b.hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// O[d_tmem] (+)= A[TMEM] * B[smem desc], bf16, fp32 accumulate.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, Desc b, uint32_t b_off16,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\t"
        "mov.b64 bd, {%2, %3};\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b.lo + b_off16), "r"(b.hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The fixed order in which the producer fills, and the MMA issuer consumes,
// the chunk ring: K_0(0), K_1(0), then per step t and slot s: V_s(t),
// K_s(t+1) (for the slots that still have tiles). fn(slot, is_v, t) returns
// false to stop the walk.
template <typename Fn>
__device__ __forceinline__ void walk_chunks(const int (&nt)[NSLOT], Fn&& fn) {
    for (int s = 0; s < NSLOT; ++s)
        if (nt[s] > 0 && !fn(s, false, 0)) return;
    const int tmax = max(nt[0], nt[1]);
    for (int t = 0; t < tmax; ++t) {
        for (int s = 0; s < NSLOT; ++s) {
            if (t < nt[s]) {
                if (!fn(s, true, t)) return;
                if (t + 1 < nt[s] && !fn(s, false, t + 1)) return;
            }
        }
    }
}

template <int D, int BQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
sparse_fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Fwd2Params prm) {
    using L = Layout2<D>;
    constexpr int NCH = L::NCHUNK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = smem + L::OFF_Q;
    uint8_t* sCH = smem + L::OFF_CH;
    Ctrl2& C = *reinterpret_cast<Ctrl2*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_k = prm.n_k;

    // The two rows of this CTA.
    int nt[NSLOT], cnt_s[NSLOT], bh_s[NSLOT], qblk_s[NSLOT];
    const int32_t* idx_row[NSLOT];
#pragma unroll
    for (int s = 0; s < NSLOT; ++s) {
        const int r = blockIdx.x * NSLOT + s;
        int c = 0;
        if (r < prm.rows) {
            if (prm.dense) {
                c = n_k;
            } else {
                c = prm.cnt[r];
                if (c < 0 || c > n_k) {
                    if (threadIdx.x == 0) record_error(SA_STATUS_DEVICE_ASSERT, 0xC000u);
                    c = c < 0 ? 0 : n_k;
                }
            }
        }
        cnt_s[s] = c;
        nt[s] = (c + 1) / 2;
        bh_s[s] = (r < prm.rows) ? r / prm.n_q : 0;
        qblk_s[s] = (r < prm.rows) ? r % prm.n_q : 0;
        idx_row[s] = (prm.dense || r >= prm.rows) ? nullptr : prm.idx + (size_t)r * n_k;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&C.q_full[s], 1);
            mbar_init(&C.s_full[s], 1);
            mbar_init(&C.p_full[s], 128);
            mbar_init(&C.o_done[s], 1);
        }
        for (int c = 0; c < NCH; ++c) {
            mbar_init(&C.ch_full[c], 1);
            mbar_init(&C.ch_empty[c], 1);
        }
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
    const uint64_t lim = prm.wait_limit_ns;

    if (warp >= 2 * 4) {
      // Control warpgroup: producer, MMA issuer, two idle warps.
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTRL_REGS));
      if (warp == PRODUCER_WARP) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_descriptor(&tmQ);
            tma_prefetch_descriptor(&tmK);
            tma_prefetch_descriptor(&tmV);
            for (int s = 0; s < NSLOT; ++s) {
                if (nt[s] == 0) continue;
                mbar_arrive_expect_tx(&C.q_full[s], L::Q_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl)
                    tma_load_3d(sQ + s * L::Q_BYTES + sl * (MROWS * 128), &tmQ, &C.q_full[s], sl * 64,
                                qblk_s[s] * BQ, bh_s[s]);
            }
        }
        int window[NSLOT] = {-1, -1};  // 32 index-list entries per slot, one per lane
        int k = 0;
        walk_chunks(nt, [&](int s, bool is_v, int t) -> bool {
            const int c = k % NCH;
            if (k >= NCH) {
                const bool w = mbar_wait_bounded(&C.ch_empty[c], ((k / NCH) - 1) & 1, abort_flag,
                                                 W_CH_EMPTY, lim);
                if (!__all_sync(0xFFFFFFFFu, w)) return false;
            }
            const int e0 = 2 * t;
            if (!is_v && (e0 & 31) == 0) {  // K of a tile comes before its V
                const int e = e0 + lane;
                window[s] = (e < cnt_s[s]) ? (prm.dense ? e : __ldg(idx_row[s] + e)) : -1;
            }
            int j0 = __shfl_sync(0xFFFFFFFFu, window[s], e0 & 31);
            int j1 = __shfl_sync(0xFFFFFFFFu, window[s], (e0 + 1) & 31);
            if (e0 + 1 >= cnt_s[s]) j1 = -1;
            if (j0 >= n_k || j0 < 0 || j1 >= n_k || j1 < -1) {
                if (lane == 0 && !is_v) record_error(SA_STATUS_DEVICE_ASSERT, 0xB000u);
                if (j0 >= n_k || j0 < 0) j0 = -1;
                if (j1 >= n_k || j1 < -1) j1 = -1;
            }
            if (lane == 0) {
                // An absent block is read at a row past N: TMA fills it with zeros.
                const int r0 = (j0 >= 0 ? j0 : n_k) * BK;
                const int r1 = (j1 >= 0 ? j1 : n_k) * BK;
                const CUtensorMap* map = is_v ? &tmV : &tmK;
                uint8_t* dst = sCH + c * L::CH_BYTES;
                mbar_arrive_expect_tx(&C.ch_full[c], L::CH_BYTES);
                for (int sl = 0; sl < L::SLABS; ++sl) {
                    uint8_t* base = dst + sl * (TILE_N * 128);
                    tma_load_3d(base, map, &C.ch_full[c], sl * 64, r0, bh_s[s]);
                    tma_load_3d(base + BK * 128, map, &C.ch_full[c], sl * 64, r1, bh_s[s]);
                }
            }
            ++k;
            return true;
        });
        // Abort path: let every copy already issued land before the CTA exits.
        if (*abort_flag && lane == 0) {
            for (int s = 0; s < NSLOT; ++s) {
                if (nt[s] == 0) continue;
                for (uint64_t t0 = globaltimer_ns();
                     !mbar_try_wait(&C.q_full[s], 0) && globaltimer_ns() - t0 < lim;) {
                }
            }
            for (int kk = (k > NCH ? k - NCH : 0); kk < k; ++kk) {
                const int c = kk % NCH;
                for (uint64_t t0 = globaltimer_ns();
                     !mbar_try_wait(&C.ch_full[c], (kk / NCH) & 1) && globaltimer_ns() - t0 < lim;) {
                }
            }
        }
      } else if (warp == MMA_WARP) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0 && (nt[0] > 0 || nt[1] > 0)) {
            constexpr uint32_t IDESC_S = make_idesc_bf16(MROWS, TILE_N, false);
            constexpr uint32_t IDESC_PV = make_idesc_bf16(MROWS, D, true);
            const Desc q_desc = desc_split(kmajor_desc(smem_u32(sQ)));
            const Desc k_desc = desc_split(kmajor_desc(smem_u32(sCH)));
            const Desc v_desc = desc_split(mnmajor_desc(smem_u32(sCH), TILE_N * 128));
            bool ok = true;
            for (int s = 0; s < NSLOT && ok; ++s)
                if (nt[s] > 0) ok = mbar_wait_bounded(&C.q_full[s], 0, abort_flag, W_Q, lim);
            int k = 0;
            if (ok) {
                walk_chunks(nt, [&](int s, bool is_v, int t) -> bool {
                    const int c = k % NCH;
                    if (!mbar_wait_bounded(&C.ch_full[c], (k / NCH) & 1, abort_flag, W_CH_FULL, lim)) {
                        ok = false;
                        return false;
                    }
                    const uint32_t c16 = (uint32_t)(c * L::CH_BYTES) >> 4;  // chunk offset, 16-byte units
                    const uint32_t tS = tmem + s * TILE_N;
                    if (!is_v) {
                        tc_fence_after();
                        const Desc qd = {q_desc.lo + ((uint32_t)(s * L::Q_BYTES) >> 4), q_desc.hi};
                        const Desc kd = {k_desc.lo + c16, k_desc.hi};
#pragma unroll
                        for (int sl = 0; sl < L::SLABS; ++sl) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                umma_ss(tS, qd, (sl * (MROWS * 128) + kk * 32) >> 4, kd,
                                        (sl * (TILE_N * 128) + kk * 32) >> 4, IDESC_S,
                                        (sl > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        umma_commit(&C.s_full[s]);
                        umma_commit(&C.ch_empty[c]);
                    } else {
                        if (!mbar_wait_bounded(&C.p_full[s], t & 1, abort_flag, W_P_FULL, lim)) {
                            ok = false;
                            return false;
                        }
                        tc_fence_after();
                        const uint32_t tO = tmem + 2 * TILE_N + s * TILE_N;
                        const Desc vd = {v_desc.lo + c16, v_desc.hi};
#pragma unroll
                        for (int kk = 0; kk < TILE_N / 16; ++kk) {
                            umma_ts(tO, tS + kk * 8, vd, (kk * 16 * 128) >> 4, IDESC_PV,
                                    (t > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&C.ch_empty[c]);
                        if (t == nt[s] - 1) umma_commit(&C.o_done[s]);
                    }
                    ++k;
                    return true;
                });
            }
            if (!ok) {
                // Abort path: wait for every MMA issued so far before TMEM is freed.
                umma_commit(&C.drain);
                for (uint64_t t0 = globaltimer_ns();
                     !mbar_try_wait(&C.drain, 0) && globaltimer_ns() - t0 < lim;) {
                }
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(SOFTMAX_REGS));
        // ------------------------------------------- softmax and epilogue
        const int s = warp / 4;                  // slot of this warpgroup
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const int row = wq * 32 + lane;          // query row within the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + s * TILE_N + lane_off;
        const uint32_t tO = tmem + 2 * TILE_N + s * TILE_N + lane_off;
        const int cnt = cnt_s[s];
        const int my_nt = nt[s];
        const int q_tok = qblk_s[s] * BQ + row;
        const bool row_valid = (row < BQ) && (q_tok < prm.N) && (blockIdx.x * NSLOT + s < prm.rows);
        const float sl2 = prm.scale_log2;
        const int32_t* lst = idx_row[s];
        // Index-list entries are loaded a tile ahead and range-checked only
        // when used, so the load latency hides behind a tile of work.
        auto block_raw = [&](int e) -> int {
            if (e >= cnt) return -1;
            return prm.dense ? e : __ldg(lst + e);
        };
        auto checked = [&](int j) -> int { return (j >= 0 && j < n_k) ? j : -1; };
        const bool want_lse = prm.lse != nullptr;
        float m_run = -INFINITY;  // running max, log2 units, as used for P
        float l_run = 0.f;        // sum of the bf16-rounded weights: normalises O
        float l_exact = 0.f;      // sum of the unrounded weights: the log-sum-exp
        bool ok = true;
        int nj0 = my_nt > 0 ? block_raw(0) : -1, nj1 = my_nt > 0 ? block_raw(1) : -1;
        for (int t = 0; t < my_nt; ++t) {
            const int j0 = checked(nj0), j1 = checked(nj1);
            if (t + 1 < my_nt) {  // next tile's blocks, loaded while this one is computed
                nj0 = block_raw(2 * t + 2);
                nj1 = block_raw(2 * t + 3);
            }
            const bool w = mbar_wait_bounded(&C.s_full[s], t & 1, abort_flag, W_S_FULL, lim);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // Valid key columns: [0, v0) from block j0, [64, 64 + v1) from j1.
            const int v0 = j0 < 0 ? 0 : min(BK, prm.N - j0 * BK);
            const int v1 = j1 < 0 ? 0 : min(BK, prm.N - j1 * BK);
            uint32_t r[TILE_N];
            tmem_ld128(tS, r);
            if (v0 < BK || v1 < BK) {  // partial tile: padding keys get -inf
#pragma unroll
                for (int c = 0; c < TILE_N; ++c) {
                    const bool valid = (c < BK) ? (c < v0) : (c - BK < v1);
                    if (!valid) r[c] = 0xFF800000u;
                }
            }
            // Row max over 8 independent chains of three-input max.
            float mc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) mc[q] = __uint_as_float(r[2 * q]);
#pragma unroll
            for (int c = 16; c < TILE_N; c += 16) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    mc[q] = max3f(mc[q], __uint_as_float(r[c + 2 * q]), __uint_as_float(r[c + 2 * q + 1]));
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) mc[q] = fmaxf(mc[q], __uint_as_float(r[2 * q + 1]));
            const float mx = fmaxf(fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])),
                                   fmaxf(fmaxf(mc[4], mc[5]), fmaxf(mc[6], mc[7]))) * sl2;
            float alpha = 1.f;
            if (mx > m_run + LAZY_RESCALE_LOG2) {
                alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mx);
                m_run = mx;
            }
            l_run *= alpha;
            l_exact *= alpha;
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            const uint64_t scale2 = f2_pack(sl2, sl2);
            const uint64_t negm2 = f2_pack(-m_use, -m_use);
            uint64_t acc[4], acc_exact[2];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = 0ull;
            acc_exact[0] = acc_exact[1] = 0ull;
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // two halves of 64 keys: P columns [32h, 32h + 32)
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int pc = 32 * h + c;  // column pair
                    // y = S * log2(e)/sqrt(d) - m for two columns at once.
                    const uint64_t y = f2_fma(f2_pack(__uint_as_float(r[2 * pc]), __uint_as_float(r[2 * pc + 1])),
                                              scale2, negm2);
                    float p0, p1;
                    if (EXP_POLY_EVERY > 0 && pc % (EXP_POLY_EVERY > 0 ? EXP_POLY_EVERY : 1) == EXP_POLY_EVERY - 1) {
                        exp2_poly_pair(y, p0, p1);
                    } else {
                        float y0, y1;
                        f2_unpack(y, y0, y1);
                        p0 = ex2_approx(y0);
                        p1 = ex2_approx(y1);
                    }
                    pk[c] = pack_bf16x2(p0, p1);
                    // Sum the bf16-rounded weights the PV product uses.
                    acc[c & 3] = f2_add(acc[c & 3], f2_pack(__uint_as_float(pk[c] << 16),
                                                            __uint_as_float(pk[c] & 0xFFFF0000u)));
                    if (want_lse) acc_exact[c & 1] = f2_add(acc_exact[c & 1], f2_pack(p0, p1));
                }
                tmem_st32_nowait(tS + 32 * h, pk);
            }
            {
                const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
                float a0, a1;
                f2_unpack(a2, a0, a1);
                l_run += a0 + a1;
                f2_unpack(f2_add(acc_exact[0], acc_exact[1]), a0, a1);
                l_exact += a0 + a1;
            }
            // O_s is stable here: S_s(t) was issued after P_s(t-1) V and its
            // completion was signalled after every earlier MMA had finished.
            if (t >= 1 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
                uint32_t o[D];
                if constexpr (D == 128) tmem_ld128(tO, o); else tmem_ld64(tO, o);
                const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll
                for (int c = 0; c < D / 2; ++c) {
                    float a0, a1;
                    f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * c]), __uint_as_float(o[2 * c + 1])), al2), a0, a1);
                    o[2 * c] = __float_as_uint(a0);
                    o[2 * c + 1] = __float_as_uint(a1);
                }
                if constexpr (D == 128) tmem_st128_nowait(tO, o); else tmem_st64_nowait(tO, o);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&C.p_full[s]);
        }

        // Epilogue: O / l, and the log-sum-exp.
        if (ok && my_nt > 0) {
            const bool w = mbar_wait_bounded(&C.o_done[s], 0, abort_flag, W_O_DONE, lim);
            ok = __all_sync(0xFFFFFFFFu, w);
            tc_fence_after();
        }
        const bool have = ok && my_nt > 0 && l_run > 0.f;
        const float inv_l = have ? 1.f / l_run : 0.f;
        const size_t out_off = ((size_t)bh_s[s] * prm.N + q_tok) * D;
        uint32_t o[D];
        if (ok && my_nt > 0) {
            if constexpr (D == 128) tmem_ld128(tO, o); else tmem_ld64(tO, o);
        } else {
#pragma unroll
            for (int e = 0; e < D; ++e) o[e] = 0u;
        }
        if (row_valid) {
            if (prm.out_f32) {
                float4* out = reinterpret_cast<float4*>(static_cast<float*>(prm.O) + out_off);
#pragma unroll
                for (int e4 = 0; e4 < D / 4; ++e4)
                    out[e4] = make_float4(__uint_as_float(o[4 * e4 + 0]) * inv_l, __uint_as_float(o[4 * e4 + 1]) * inv_l,
                                          __uint_as_float(o[4 * e4 + 2]) * inv_l, __uint_as_float(o[4 * e4 + 3]) * inv_l);
            } else {
                uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.O) + out_off);
#pragma unroll
                for (int e8 = 0; e8 < D / 8; ++e8) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(o[8 * e8 + 0]) * inv_l, __uint_as_float(o[8 * e8 + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(o[8 * e8 + 2]) * inv_l, __uint_as_float(o[8 * e8 + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(o[8 * e8 + 4]) * inv_l, __uint_as_float(o[8 * e8 + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(o[8 * e8 + 6]) * inv_l, __uint_as_float(o[8 * e8 + 7]) * inv_l);
                    out[e8] = v;
                }
            }
        }
        if (row_valid && prm.lse) {
            prm.lse[(size_t)bh_s[s] * prm.N + q_tok] =
                have ? (m_run + __log2f(l_exact)) * 0.69314718055994531f : -INFINITY;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace fwd2
}  // namespace sa
