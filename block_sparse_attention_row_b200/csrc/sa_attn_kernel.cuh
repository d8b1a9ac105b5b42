// sa_attn_kernel.cuh - step 4 of the path: block-sparse FlashAttention-style
// forward over the kept (query block, key block) tiles only, for sm_100a.
//
// Method: "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
// Masking and Distillation Fine-Tuning" (gist.science summary) §2C Efficient
// Kernel Implementation: the tensors are split into tiles, the hybrid mask is
// applied per block, and the matmuls and softmax of masked tiles are skipped.
// Here a masked tile is never loaded, multiplied or exponentiated: each query
// block walks only its own kept-block list.
//
// Persistent kernel: one CTA per SM runs two independent pipelines ("slots").
// Slot s of CTA b serves the query-block rows r = 2b + s, 2b + s + 2G, ...
// (G CTAs), one after the other, so that a row's start (its Q tile, its first
// K tile) and end (the epilogue) overlap the neighbouring rows' work and the
// other slot's matmuls. 384 threads in four roles:
//   warps 8, 11  TMA producers of slot 0 and slot 1: the Q tile of each row,
//                then the row's K and V tiles (two kept key blocks = 128 keys
//                per tile) gathered by its index list into the slot's ring of
//                chunks, in the order K(0), V(0), K(1), V(1), ...;
//   warps 9, 10  tcgen05 issuers (one thread each) of slot 0 and slot 1:
//                S_s = Q_s K(t)^T into TMEM; O_s += P_s V(t) with P_s read from
//                TMEM where the softmax wrote it over S_s; S_s(t+1) follows
//                P_s V(t) (the tensor pipe executes one thread's MMAs in order).
//                A batch of MMAs is issued whole under a ticket lock, so the
//                two slots' batches reach the tensor pipe one after the other
//                and the slots settle into alternation: one slot's softmax runs
//                while the other slot's matmuls do;
//   warps 0-3    softmax of slot 0, warps 4-7 softmax of slot 1: one query row
//                per thread (one TMEM lane), base-2 online softmax (a tile's
//                own max is taken only on a row's first tile and when its
//                weights against the running max would pass 2^64; O is then
//                rescaled), then each row's epilogue through a staging tile
//                and TMA stores.
// The control warpgroup (8-11) hands most of its registers to the two
// softmax warpgroups (setmaxnreg).
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d),
// O_1 [384,384+d); P_s (bf16 pairs) overwrites the first 64 columns of S_s.
// Tensor-core shapes: S tile M=128 x N=128 x K=d (A, B from shared memory);
// PV tile M=128 x N=d x K=128 (A from TMEM, B = V from shared memory).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"
#include "sa_mask_kernels.cuh"

namespace sa {
namespace attn {

constexpr int BK = 64;           // key block (tokens)
constexpr int TILE_N = 128;      // keys per tile: two kept key blocks
constexpr int MROWS = 128;       // query rows per MMA tile
constexpr int NSLOT = 2;         // independent row pipelines per CTA
constexpr int NUM_THREADS = 384;   // softmax warpgroups 0-1, control warpgroup 2
constexpr int PRODUCER_WARP0 = 8;  // slot 0; slot 1's producer is warp 11
constexpr int PRODUCER_WARP1 = 11;
constexpr int MMA_WARP = 9;        // slot 0; slot 1's issuer is warp 10
// Register split (setmaxnreg): the kernel launches with LAUNCH_REGS per thread
// (384 x 168 = 64512 registers); the control warpgroup gives back down to
// CTRL_REGS and the two softmax warpgroups take the rest:
// 128 x 56 + 256 x 224 = 64512.
constexpr int LAUNCH_REGS = 168;
constexpr int CTRL_REGS = 56;
constexpr int SOFTMAX_REGS = 224;
static_assert(128 * CTRL_REGS + 256 * SOFTMAX_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 512;
// A tile's weights 2^(S log2(e)/sqrt(d) - m_run) are used against the running
// max as long as their sum stays at or below 2^64 (so every weight does); O
// and l then stay far inside the fp32 range for any realistic V. Past that,
// or on a row's first tile, the tile's own max is taken.
constexpr float MAX_TILE_SUM = 18446744073709551616.0f;   // 2^64
// Serialise the two issuers' MMA batches (see above).
constexpr bool ISSUE_LOCK = true;
constexpr int MAX_CH = 4;

// Where a bounded wait gave up (reported in the device error record).
enum WaitSite : unsigned int {
    W_CH_EMPTY = 0xE001, W_Q = 0xE002, W_CH_FULL = 0xE003, W_P_FULL = 0xE004,
    W_S_FULL = 0xE005, W_O_FULL = 0xE006, W_Q_EMPTY = 0xE007, W_LOCK = 0xE008, W_STG = 0xE009,
    W_GRID_POOL = 0xE00A, W_GRID_SELECT = 0xE00B
};

// FP8: Q and K are e4m3 codes (one byte per element, 128 channels per
// 128-byte slab) with per-block scales; V stays bf16.
template <int D, bool FP8 = false>
struct Layout {
    static constexpr int SLABS = D / 64;                 // 64-channel (128-byte) bf16 slabs: V, O
    static constexpr int QK_SLABS = FP8 ? D / 128 : D / 64;   // 128-byte slabs of Q and K
    static constexpr int QK_CH = FP8 ? 128 : 64;         // channels per Q/K slab
    static constexpr int Q_BYTES = MROWS * D * (FP8 ? 1 : 2);   // one Q tile
    static constexpr int K_BYTES = TILE_N * D * (FP8 ? 1 : 2);  // one K tile
    static constexpr int CH_BYTES = TILE_N * D * 2;      // one chunk slot: a V tile or a K tile
    static_assert(!FP8 || D == 128, "the FP8 path is built for d = 128");
    static constexpr int NCH = (D == 128) ? 2 : 4;       // chunk ring depth per slot
    static constexpr int SLOT_BYTES = Q_BYTES + NCH * CH_BYTES;
    // Per slot, the staging tile of the bf16 epilogue: 128 rows x 64 channels.
    static constexpr int STG_BYTES = MROWS * 128;
    static constexpr int OFF_STG = NSLOT * SLOT_BYTES;
    static constexpr int OFF_CTRL = OFF_STG + NSLOT * STG_BYTES;
    static constexpr int CTRL_BYTES = 512;
    static constexpr int DYN_BYTES = OFF_CTRL + CTRL_BYTES + 1024;
    static_assert(NCH <= MAX_CH, "chunk ring too deep");
    static_assert(NCH % 2 == 0, "K and V tiles alternate through the ring");
    static_assert(DYN_BYTES <= 232448, "shared memory budget");
    static_assert(DYN_BYTES > 116 * 1024, "one CTA per SM (TMEM is allocated whole)");
};

struct SlotBars {
    uint64_t q_full, q_empty;
    uint64_t ch_full[MAX_CH], ch_empty[MAX_CH];
    uint64_t s_full;   // S_s(t) is in TMEM (and every earlier MMA of the slot is done)
    uint64_t p_full;   // the softmax wrote P_s(t) (and rescaled O_s if it had to)
    uint64_t o_full;   // the row's last P V is done
    uint64_t drain;    // abort path: completion of every MMA the slot's issuer issued
    uint64_t stg_full; // the four softmax warps wrote the staging tile
    uint64_t stg_free; // the staging tile's last store has read it
};

struct Ctrl {
    SlotBars sb[NSLOT];
    uint32_t tmem_base;
    int abort_flag;
    int ticket_next;
    int ticket_serving;
};

struct Params {
    const int32_t* cnt;  // [BH * n_q]
    const int32_t* idx;  // [BH * n_q, n_k]
    void* O;             // [BH, N, D], bf16 or fp32 (out_f32)
    float* lse;          // [BH, N] or null
    int N, n_q, n_k, rows;
    int dense;           // 1: every key block, no index list
    int out_f32;         // 1: O is fp32, 0: bf16 (round to nearest even)
    float scale_log2;    // log2(e) / sqrt(d)
    unsigned long long wait_limit_ns;
    // Failure-detection test only: 1 makes the producer of slot 0 of CTA 0
    // skip the copy of its first K tile (nothing is armed or issued for it),
    // so that the waits depending on it run out. 0 in every normal launch.
    int withhold_first_k;
    // FP8 path: per-block scales of the Q and K codes (null otherwise).
    const float* q_scale;   // [BH * n_q]
    const float* k_scale;   // [BH * n_k]
    // Single-launch path only: the mask phases' inputs and outputs. cnt and
    // idx above are then the buffers these phases write (cnt_w, idx_w).
    const void* q_in;       // bf16 Q, K [BH, N, D]
    const void* k_in;
    float* qbar;            // [BH * n_q, D] block means (workspace)
    float* kbar;            // [BH * n_k, D]
    unsigned int* grid_ctr; // grid-barrier counter, zeroed before the launch
    int32_t* cnt_w;
    int32_t* idx_w;
    int BH, bq, kc;
    double p;
    float score_scale;      // 1/sqrt(d)
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
    return make_sdesc_sw128(addr, 16u, 1024u);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr, uint32_t slab_bytes) {
    return make_sdesc_sw128(addr, slab_bytes, 1024u);
}

// Shared-memory descriptors as (low, high) word pairs: moving the start
// address by a byte offset adds offset >> 4 to the low word (offsets stay
// below 2^18 bytes, so the 14-bit field never carries).
struct Desc {
    uint32_t lo, hi;
};
__device__ __forceinline__ Desc desc_split(uint64_t d) {
    return {static_cast<uint32_t>(d), static_cast<uint32_t>(d >> 32)};
}
__device__ __forceinline__ uint64_t desc_at(Desc d, uint32_t off16) {
    return ((uint64_t)d.hi << 32) | (uint64_t)(d.lo + off16);
}

// N consecutive MMAs into one accumulator, issued back to back from one asm
// statement so that no other instruction sits between two issues. The first
// MMA overwrites D unless acc0 is set; the others accumulate.
template <int N>
__device__ __forceinline__ void umma_ss_batch(uint32_t d_tmem, const uint64_t (&a)[N], const uint64_t (&b)[N],
                                              uint32_t idesc, uint32_t acc0);
template <>
__device__ __forceinline__ void umma_ss_batch<8>(uint32_t d, const uint64_t (&a)[8], const uint64_t (&b)[8],
                                                 uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %18, 0;\n\t"
        "setp.eq.b32 p1, %17, %17;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %17, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %17, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %17, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %17, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %17, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %17, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %17, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %17, p1;\n\t}" ::"r"(d),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]), "l"(a[7]),
        "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]),
        "r"(idesc), "r"(acc0)
        : "memory");
}
template <>
__device__ __forceinline__ void umma_ss_batch<4>(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                                 uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %10, 0;\n\t"
        "setp.eq.b32 p1, %9, %9;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, p1;\n\t}" ::"r"(d),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
        "r"(idesc), "r"(acc0)
        : "memory");
}

// Four SS MMAs of kind::f8f6f4 (e4m3 A and B, K = 32 each) into one accumulator.
__device__ __forceinline__ void umma_ss_batch_f8x4(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                                   uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %10, 0;\n\t"
        "setp.eq.b32 p1, %9, %9;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %5, %9, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %2, %6, %9, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %3, %7, %9, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %4, %8, %9, p1;\n\t}" ::"r"(d),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
        "r"(idesc), "r"(acc0)
        : "memory");
}

// Eight TS MMAs (A from TMEM columns a_tmem + 8i, B descriptors b[i]) into D.
__device__ __forceinline__ void umma_ts_batch8(uint32_t d, uint32_t a_tmem, const uint64_t (&b)[8],
                                               uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 a;\n\t"
        "setp.ne.b32 p0, %11, 0;\n\t"
        "setp.eq.b32 p1, %10, %10;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %10, p0;\n\t"
        "add.u32 a, %1, 8;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %3, %10, p1;\n\t"
        "add.u32 a, %1, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %4, %10, p1;\n\t"
        "add.u32 a, %1, 24;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %5, %10, p1;\n\t"
        "add.u32 a, %1, 32;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %6, %10, p1;\n\t"
        "add.u32 a, %1, 40;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %7, %10, p1;\n\t"
        "add.u32 a, %1, 48;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %8, %10, p1;\n\t"
        "add.u32 a, %1, 56;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], %9, %10, p1;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]),
        "l"(b[7]), "r"(idesc), "r"(acc0)
        : "memory");
}

// The lists are read through the read-only path, except on the single-launch
// path (CG), where this launch wrote them: there they are read through L2.
template <bool CG>
__device__ __forceinline__ int ld_list(const int32_t* p) {
    if constexpr (CG) return __ldcg(p);
    else return __ldg(p);
}

// Kept-block count of a row as stored (loaded a row ahead, checked at use, so
// that the load's latency is not waited for until then).
template <bool CG>
__device__ __forceinline__ int raw_count(const Params& prm, int r) {
    return prm.dense ? prm.n_k : ld_list<CG>(prm.cnt + r);
}
// A count range-checked (a bad count is recorded and clamped).
__device__ __forceinline__ int checked_count(const Params& prm, int c) {
    if (c < 0 || c > prm.n_k) {
        record_error(SA_STATUS_DEVICE_ASSERT, 0xC000u);
        c = c < 0 ? 0 : prm.n_k;
    }
    return c;
}

// Index-list entry e of row r for this lane, -1 past the row's count.
template <bool CG>
__device__ __forceinline__ int list_entry(const Params& prm, int r, int cnt, int e) {
    if (e >= cnt) return -1;
    return prm.dense ? e : ld_list<CG>(prm.idx + (size_t)r * prm.n_k + e);
}

// Index-list entry e of row r without the count check (-1 past n_k): loaded a
// row ahead, before the row's count is known, and masked with it at use.
template <bool CG>
__device__ __forceinline__ int raw_entry(const Params& prm, int r, int e) {
    if (r >= prm.rows || e >= prm.n_k) return -1;
    return prm.dense ? e : ld_list<CG>(prm.idx + (size_t)r * prm.n_k + e);
}

// Ticket lock that hands the tensor pipe to one issuer's batch at a time.
__device__ __forceinline__ bool issue_acquire(Ctrl& C, int& ticket, volatile int* abort_flag, uint64_t lim) {
    if (!ISSUE_LOCK) return true;
    ticket = atomicAdd(&C.ticket_next, 1);
    volatile int* serving = &C.ticket_serving;
    if (*serving == ticket) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (*serving == ticket) return true;
        if ((it & 255u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > lim) {
                record_error(SA_STATUS_TIMEOUT, W_LOCK);
                *abort_flag = 1;
                return false;
            }
        }
    }
}
__device__ __forceinline__ void issue_release(Ctrl& C, int ticket) {
    if (!ISSUE_LOCK) return;
    *reinterpret_cast<volatile int*>(&C.ticket_serving) = ticket + 1;
}

template <int D, int BQ, bool FP8 = false, bool FUSED = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const Params prm) {
    using L = Layout<D, FP8>;
    constexpr int NCH = L::NCH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    Ctrl& C = *reinterpret_cast<Ctrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &C.abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_k = prm.n_k;
    const int P = NSLOT * gridDim.x;   // row pipelines in the grid

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            SlotBars& B = C.sb[s];
            mbar_init(&B.q_full, 1);
            mbar_init(&B.q_empty, 1);
            for (int c = 0; c < NCH; ++c) {
                mbar_init(&B.ch_full[c], 1);
                mbar_init(&B.ch_empty[c], 1);
            }
            mbar_init(&B.s_full, 1);
            mbar_init(&B.p_full, 4);   // one arrival per softmax warp
            mbar_init(&B.o_full, 1);
            mbar_init(&B.drain, 1);
            mbar_init(&B.stg_full, 4);   // one arrival per softmax warp
            mbar_init(&B.stg_free, 1);
        }
        C.abort_flag = 0;
        C.ticket_next = 0;
        C.ticket_serving = 0;
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

    if constexpr (FUSED) {
        // The mask, in this launch (cooperative: every CTA is resident): the
        // block means, a grid barrier, the scores and kept lists of every row,
        // a grid barrier; then the attention below reads the lists. Shared
        // memory below the control block serves as the phases' scratch.
        sa::mask::fused_pool_phase<D>(static_cast<const __nv_bfloat16*>(prm.q_in),
                                      static_cast<const __nv_bfloat16*>(prm.k_in), prm.qbar, prm.kbar, prm.BH,
                                      prm.N, prm.bq, BK, prm.n_q, n_k, reinterpret_cast<float*>(smem));
        if (sa::mask::grid_barrier(prm.grid_ctr, gridDim.x, lim, abort_flag, W_GRID_POOL))
            sa::mask::fused_select_phase<D>(prm.qbar, prm.kbar, prm.BH, prm.n_q, n_k, prm.score_scale, prm.kc,
                                            prm.p, prm.cnt_w, prm.idx_w, smem);
        // The scratch is rewritten by TMA and read by the MMAs (async proxy).
        fence_proxy_async_smem();
        sa::mask::grid_barrier(prm.grid_ctr, 2 * gridDim.x, lim, abort_flag, W_GRID_SELECT);
    }

    if (FUSED && *abort_flag) {
        // A grid barrier ran out: no attention (nothing was issued).
    } else if (warp >= 8) {
      // Control warpgroup: producers and MMA issuers.
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTRL_REGS));
      if (warp == PRODUCER_WARP0 || warp == PRODUCER_WARP1) {
        // ------------------------------------------------------ TMA producer
        const int s = (warp == PRODUCER_WARP0) ? 0 : 1;
        SlotBars& B = C.sb[s];
        uint8_t* sQ = smem + s * L::SLOT_BYTES;
        uint8_t* sCH = sQ + L::Q_BYTES;
        if (lane == 0) {
            tma_prefetch_descriptor(&tmQ);
            tma_prefetch_descriptor(&tmK);
            tma_prefetch_descriptor(&tmV);
        }
        int k = 0, kq = 0;
        bool ok = true;
        // The next row's count and first 64 index entries are loaded a row ahead.
        const int r_first = blockIdx.x * NSLOT + s;
        int cnt_next = r_first < prm.rows ? raw_count<FUSED>(prm, r_first) : 0;
        int raw0_next = raw_entry<FUSED>(prm, r_first, lane), raw1_next = raw_entry<FUSED>(prm, r_first, 32 + lane);
        for (int r = r_first; ok && r < prm.rows; r += P) {
            const int cnt = checked_count(prm, cnt_next);
            const int raw0 = raw0_next, raw1 = raw1_next;
            if (r + P < prm.rows) {
                cnt_next = raw_count<FUSED>(prm, r + P);
                raw0_next = raw_entry<FUSED>(prm, r + P, lane);
                raw1_next = raw_entry<FUSED>(prm, r + P, 32 + lane);
            }
            const int nt = (cnt + 1) / 2;
            if (nt == 0) continue;
            const int bh = r / prm.n_q, qb = r % prm.n_q;
            if (kq > 0) {
                const bool w = mbar_wait_bounded(&B.q_empty, (kq - 1) & 1, abort_flag, W_Q_EMPTY, lim);
                if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&B.q_full, L::Q_BYTES);
                for (int sl = 0; sl < L::QK_SLABS; ++sl)
                    tma_load_3d(sQ + sl * (MROWS * 128), &tmQ, &B.q_full, sl * L::QK_CH, qb * BQ, bh);
                const int rn = r + P;   // the slot's next row: its Q tile into L2 now
                if (rn < prm.rows)
                    for (int sl = 0; sl < L::QK_SLABS; ++sl)
                        tma_prefetch_l2_3d(&tmQ, sl * L::QK_CH, (rn % prm.n_q) * BQ, rn / prm.n_q);
            }
            ++kq;
            int window = lane < cnt ? raw0 : -1;                 // entries [0, 32)
            int window_next = 32 + lane < cnt ? raw1 : -1;       // entries [32, 64)
            for (int t = 0; t < nt; ++t) {
                const int e0 = 2 * t;
                if (e0 > 0 && (e0 & 31) == 0) {
                    window = window_next;
                    window_next = list_entry<FUSED>(prm, r, cnt, e0 + 32 + lane);
                }
                int j0 = __shfl_sync(0xFFFFFFFFu, window, e0 & 31);
                int j1 = __shfl_sync(0xFFFFFFFFu, window, (e0 + 1) & 31);
                if (e0 + 1 >= cnt) j1 = -1;
                if (j0 >= n_k || j0 < 0 || j1 >= n_k || j1 < -1) {
                    if (lane == 0) record_error(SA_STATUS_DEVICE_ASSERT, 0xB000u);
                    if (j0 >= n_k || j0 < 0) j0 = -1;
                    if (j1 >= n_k || j1 < -1) j1 = -1;
                }
                // An absent block is read at a row past N: TMA fills it with zeros.
                const int r0 = (j0 >= 0 ? j0 : n_k) * BK;
                const int r1 = (j1 >= 0 ? j1 : n_k) * BK;
#pragma unroll
                for (int kv = 0; kv < 2; ++kv) {   // K(t), then V(t)
                    const int c = k % NCH;
                    if (k >= NCH) {
                        const bool w = mbar_wait_bounded(&B.ch_empty[c], ((k / NCH) - 1) & 1, abort_flag,
                                                         W_CH_EMPTY, lim);
                        if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }
                    }
                    const bool withheld = prm.withhold_first_k && k == 0 && s == 0 && blockIdx.x == 0;
                    if (lane == 0 && !withheld) {
                        const CUtensorMap* map = kv ? &tmV : &tmK;
                        uint8_t* dst = sCH + c * L::CH_BYTES;
                        const int nsl = kv ? L::SLABS : L::QK_SLABS;
                        const int sch = kv ? 64 : L::QK_CH;
                        mbar_arrive_expect_tx(&B.ch_full[c], kv ? L::CH_BYTES : L::K_BYTES);
                        for (int sl = 0; sl < nsl; ++sl) {
                            uint8_t* base = dst + sl * (TILE_N * 128);
                            tma_load_3d(base, map, &B.ch_full[c], sl * sch, r0, bh);
                            tma_load_3d(base + BK * 128, map, &B.ch_full[c], sl * sch, r1, bh);
                        }
                    }
                    ++k;
                }
                if (!ok) break;
            }
        }
        // Abort path: let every copy already issued land before the CTA exits.
        if (*abort_flag && lane == 0) {
            if (kq > 0)
                for (uint64_t t0 = globaltimer_ns();
                     !mbar_try_wait(&B.q_full, (kq - 1) & 1) && globaltimer_ns() - t0 < lim;) {
                }
            for (int kk = (k > NCH ? k - NCH : 0); kk < k; ++kk) {
                const int c = kk % NCH;
                for (uint64_t t0 = globaltimer_ns();
                     !mbar_try_wait(&B.ch_full[c], (kk / NCH) & 1) && globaltimer_ns() - t0 < lim;) {
                }
            }
        }
      } else {
        // ------------------------------------------------- MMA issuers
        const int s = warp - MMA_WARP;
        SlotBars& B = C.sb[s];
        if (lane == 0) {
            constexpr uint32_t IDESC_S = FP8 ? make_idesc_e4m3(MROWS, TILE_N) : make_idesc_bf16(MROWS, TILE_N, false);
            constexpr uint32_t IDESC_PV = make_idesc_bf16(MROWS, D, true);
            uint8_t* sQ = smem + s * L::SLOT_BYTES;
            uint8_t* sCH = sQ + L::Q_BYTES;
            const Desc q_desc = desc_split(kmajor_desc(smem_u32(sQ)));
            const Desc k_desc = desc_split(kmajor_desc(smem_u32(sCH)));
            const Desc v_desc = desc_split(mnmajor_desc(smem_u32(sCH), TILE_N * 128));
            const uint32_t tS = tmem + s * TILE_N;
            const uint32_t tO = tmem + 2 * TILE_N + s * TILE_N;
            // S_s = Q_s K^T from the K tile in chunk c.
            auto issue_s = [&](int c) {
                const Desc kd = {k_desc.lo + ((uint32_t)(c * L::CH_BYTES) >> 4), k_desc.hi};
                uint64_t ad[L::QK_SLABS * 4], bd[L::QK_SLABS * 4];
#pragma unroll
                for (int sl = 0; sl < L::QK_SLABS; ++sl)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        ad[sl * 4 + kk] = desc_at(q_desc, (sl * (MROWS * 128) + kk * 32) >> 4);
                        bd[sl * 4 + kk] = desc_at(kd, (sl * (TILE_N * 128) + kk * 32) >> 4);
                    }
                if constexpr (FP8) umma_ss_batch_f8x4(tS, ad, bd, IDESC_S, 0u);
                else umma_ss_batch<L::QK_SLABS * 4>(tS, ad, bd, IDESC_S, 0u);
            };
            auto wait_chunk = [&](int kk) -> bool {
                return mbar_wait_spin(&B.ch_full[kk % NCH], (kk / NCH) & 1, abort_flag, W_CH_FULL, lim);
            };
            int k = 0, g = 0, kq = 0, ticket = 0;
            bool ok = true;
            const int r_first = blockIdx.x * NSLOT + s;
            int cnt_next = r_first < prm.rows ? raw_count<FUSED>(prm, r_first) : 0;   // a row ahead
            for (int r = r_first; ok && r < prm.rows; r += P) {
                const int nt = (checked_count(prm, cnt_next) + 1) / 2;
                if (r + P < prm.rows) cnt_next = raw_count<FUSED>(prm, r + P);
                if (nt == 0) continue;
                if (!mbar_wait_bounded(&B.q_full, kq & 1, abort_flag, W_Q, lim) || !wait_chunk(k)) {
                    ok = false;
                    break;
                }
                ++kq;
                tc_fence_after();
                if (!issue_acquire(C, ticket, abort_flag, lim)) { ok = false; break; }
                issue_s(k % NCH);
                issue_release(C, ticket);
                umma_commit(&B.s_full);
                umma_commit(&B.ch_empty[k % NCH]);
                if (nt == 1) umma_commit(&B.q_empty);
                ++k;
                for (int t = 0; t < nt; ++t) {
                    const bool more = t + 1 < nt;
                    // V(t) landed, K(t+1) landed (both normally long before), and
                    // P_s(t) written (and O_s rescaled): the batch goes out as soon
                    // as the softmax hands P over.
                    if (!wait_chunk(k) || (more && !wait_chunk(k + 1)) ||
                        !mbar_wait_spin(&B.p_full, g & 1, abort_flag, W_P_FULL, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int cv = k % NCH;
                    const Desc vd = {v_desc.lo + ((uint32_t)(cv * L::CH_BYTES) >> 4), v_desc.hi};
                    uint64_t bv[TILE_N / 16];
#pragma unroll
                    for (int kk = 0; kk < TILE_N / 16; ++kk) bv[kk] = desc_at(vd, (kk * 16 * 128) >> 4);
                    if (!issue_acquire(C, ticket, abort_flag, lim)) { ok = false; break; }
                    umma_ts_batch8(tO, tS, bv, IDESC_PV, t > 0 ? 1u : 0u);
                    if (more) issue_s((k + 1) % NCH);
                    issue_release(C, ticket);
                    // Commits after the S MMAs also cover the P V before them, so
                    // the V chunk is released no later than it would be alone.
                    umma_commit(&B.ch_empty[cv]);
                    if (more) {
                        umma_commit(&B.s_full);
                        umma_commit(&B.ch_empty[(k + 1) % NCH]);
                        if (t + 2 == nt) umma_commit(&B.q_empty);
                    } else {
                        umma_commit(&B.o_full);
                    }
                    k += more ? 2 : 1;
                    ++g;
                }
            }
            if (!ok) {
                // Abort path: wait for every MMA this thread issued before TMEM is freed.
                umma_commit(&B.drain);
                for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(&B.drain, 0) && globaltimer_ns() - t0 < lim;) {
                }
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(SOFTMAX_REGS));
        // ------------------------------------------- softmax and epilogue
        const int s = warp / 4;                  // slot of this warpgroup
        SlotBars& B = C.sb[s];
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const int row = wq * 32 + lane;          // query row within the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + s * TILE_N + lane_off;
        const uint32_t tO = tmem + 2 * TILE_N + s * TILE_N + lane_off;
        const float sl2 = prm.scale_log2;
        const bool want_lse = prm.lse != nullptr;
        auto checked = [&](int j) -> int { return (j >= 0 && j < n_k) ? j : -1; };
        int g = 0, rowc = 0;
        int npass = 0;                            // staging-tile stores of this slot so far
        bool ok = true;
        // The next row's count and first 64 index entries are loaded a row ahead.
        const int r_first = blockIdx.x * NSLOT + s;
        int cnt_next = r_first < prm.rows ? raw_count<FUSED>(prm, r_first) : 0;
        int raw0_next = raw_entry<FUSED>(prm, r_first, lane), raw1_next = raw_entry<FUSED>(prm, r_first, 32 + lane);
        for (int r = r_first; ok && r < prm.rows; r += P) {
            const int cnt = checked_count(prm, cnt_next);
            const int raw0 = raw0_next, raw1 = raw1_next;
            if (r + P < prm.rows) {
                cnt_next = raw_count<FUSED>(prm, r + P);
                raw0_next = raw_entry<FUSED>(prm, r + P, lane);
                raw1_next = raw_entry<FUSED>(prm, r + P, 32 + lane);
            }
            const int nt = (cnt + 1) / 2;
            const int bh = r / prm.n_q, qb = r % prm.n_q;
            const int q_tok = qb * BQ + row;
            const bool row_valid = (row < BQ) && (q_tok < prm.N);
            const size_t out_off = ((size_t)bh * prm.N + q_tok) * D;
            // FP8: scale of this query block's Q codes (the key blocks' scales are read per tile).
            const float row_sq = FP8 ? __ldg(prm.q_scale + (size_t)bh * prm.n_q + qb) : 1.f;
            float m_run = -INFINITY;  // running max, log2 units, as used for P
            float l_run = 0.f;        // sum of the bf16-rounded weights: normalises O
            float l_exact = 0.f;      // sum of the unrounded weights: the log-sum-exp
            // Index-list entries, 32 at a time (one per lane), one window ahead.
            int window = lane < cnt ? raw0 : -1;
            int window_next = 32 + lane < cnt ? raw1 : -1;
            for (int t = 0; t < nt; ++t) {
                const int e0 = 2 * t;
                if (e0 > 0 && (e0 & 31) == 0) {
                    window = window_next;
                    window_next = list_entry<FUSED>(prm, r, cnt, e0 + 32 + lane);
                }
                const int j0 = checked(__shfl_sync(0xFFFFFFFFu, window, e0 & 31));
                const int j1 = (e0 + 1 < cnt) ? checked(__shfl_sync(0xFFFFFFFFu, window, (e0 + 1) & 31)) : -1;
                const bool w = mbar_wait_bounded(&B.s_full, g & 1, abort_flag, W_S_FULL, lim);
                if (!__all_sync(0xFFFFFFFFu, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Valid key columns: [0, v0) from block j0, [64, 64 + v1) from j1.
                const int v0 = j0 < 0 ? 0 : min(BK, prm.N - j0 * BK);
                const int v1 = j1 < 0 ? 0 : min(BK, prm.N - j1 * BK);
                // Exponent scale of each half of the tile: log2(e)/sqrt(d), times
                // the Q and K block scales on the FP8 path (kept positive so that
                // -inf padding stays -inf; a zero scale only occurs for an
                // all-zero block, whose codes, and scores, are 0).
                float sc0 = sl2, sc1 = sl2;
                if constexpr (FP8) {
                    const float* ks = prm.k_scale + (size_t)bh * n_k;
                    sc0 = sl2 * fmaxf(row_sq * (j0 >= 0 ? __ldg(ks + j0) : 1.f), 1e-30f);
                    sc1 = sl2 * fmaxf(row_sq * (j1 >= 0 ? __ldg(ks + j1) : 1.f), 1e-30f);
                }
                // The weights of a tile are taken against the running max m_run
                // as it stands, without the tile's own max: fp32 and bf16 hold
                // weights up to 2^MAX_WEIGHT_LOG2 without loss of relative
                // precision, so the max is only needed when a tile's weights
                // would exceed that (checked on their sum, which also catches a
                // non-finite score), and on a row's first tile. Then the tile's
                // max is taken, m_run raised, and the tile's weights recomputed
                // from S_s(t), still in TMEM; O_s and the sums are rescaled.
                float alpha = 1.f;
                uint32_t pk[TILE_N / 2];
                float l_t = 0.f, le_t = 0.f;
                for (bool with_max = (t == 0);; with_max = true) {
                    uint32_t rr[TILE_N];
                    tmem_ld128(tS, rr);
                    if (v0 < BK || v1 < BK) {  // partial tile: padding keys get -inf
#pragma unroll
                        for (int c = 0; c < TILE_N; ++c) {
                            const bool valid = (c < BK) ? (c < v0) : (c - BK < v1);
                            if (!valid) rr[c] = 0xFF800000u;
                        }
                    }
                    if (FP8 && with_max) {
                        // Max of each half (its own scale), 8 chains of three-input max each.
                        float mh[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            float mc[8];
#pragma unroll
                            for (int q = 0; q < 8; ++q) mc[q] = __uint_as_float(rr[64 * h + 2 * q]);
#pragma unroll
                            for (int c = 64 * h + 16; c < 64 * h + 64; c += 16) {
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    mc[q] = max3f(mc[q], __uint_as_float(rr[c + 2 * q]), __uint_as_float(rr[c + 2 * q + 1]));
                            }
#pragma unroll
                            for (int q = 0; q < 8; ++q) mc[q] = fmaxf(mc[q], __uint_as_float(rr[64 * h + 2 * q + 1]));
                            mh[h] = fmaxf(fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])),
                                          fmaxf(fmaxf(mc[4], mc[5]), fmaxf(mc[6], mc[7])));
                        }
                        const float mx = fmaxf(mh[0] * sc0, mh[1] * sc1);
                        if (t == 0) {
                            m_run = mx;
                        } else if (mx > m_run) {
                            alpha = ex2_approx(m_run - mx);
                            m_run = mx;
                        }
                    } else if (with_max) {
                        // Row max over 8 independent chains of three-input max.
                        float mc[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) mc[q] = __uint_as_float(rr[2 * q]);
#pragma unroll
                        for (int c = 16; c < TILE_N; c += 16) {
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                mc[q] = max3f(mc[q], __uint_as_float(rr[c + 2 * q]), __uint_as_float(rr[c + 2 * q + 1]));
                        }
#pragma unroll
                        for (int q = 0; q < 8; ++q) mc[q] = fmaxf(mc[q], __uint_as_float(rr[2 * q + 1]));
                        const float mx = fmaxf(fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])),
                                               fmaxf(fmaxf(mc[4], mc[5]), fmaxf(mc[6], mc[7]))) * sl2;
                        if (t == 0) {
                            m_run = mx;
                        } else if (mx > m_run) {
                            alpha = ex2_approx(m_run - mx);
                            m_run = mx;
                        }
                    }
                    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                    const uint64_t scale2 = f2_pack(sc0, sc0);
                    const uint64_t scale2_hi = f2_pack(sc1, sc1);   // the second half (equal unless FP8)
                    const uint64_t negm2 = f2_pack(-m_use, -m_use);
                    uint64_t acc[4], acc_exact[2];
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[q] = 0ull;
                    acc_exact[0] = acc_exact[1] = 0ull;
                    // The exponentials run as independent stages over the whole row
                    // (arguments, then MUFU, then packing, then sums) so that the
                    // scheduler always has many independent instructions in flight.
                    float pe[TILE_N];
#pragma unroll
                    for (int pc = 0; pc < TILE_N / 2; ++pc) {
                        // y = S * log2(e)/sqrt(d) - m for two columns at once.
                        const uint64_t y = f2_fma(f2_pack(__uint_as_float(rr[2 * pc]), __uint_as_float(rr[2 * pc + 1])),
                                                  (FP8 && pc >= TILE_N / 4) ? scale2_hi : scale2, negm2);
                        f2_unpack(y, pe[2 * pc], pe[2 * pc + 1]);
                    }
#pragma unroll
                    for (int c = 0; c < TILE_N; ++c) pe[c] = ex2_approx(pe[c]);
#pragma unroll
                    for (int pc = 0; pc < TILE_N / 2; ++pc) pk[pc] = pack_bf16x2(pe[2 * pc], pe[2 * pc + 1]);
#pragma unroll
                    for (int pc = 0; pc < TILE_N / 2; ++pc) {
                        // Sum the bf16-rounded weights the P V product uses, so
                        // that O / l is exactly a convex combination of V rows
                        // (normalising by the unrounded sum, as FlashAttention
                        // does, measured a max-abs error of 1.01e-2 on the Mid
                        // workload against the oracle, past the 1e-2 bound).
                        acc[pc & 3] = f2_add(acc[pc & 3], f2_pack(__uint_as_float(pk[pc] << 16),
                                                                  __uint_as_float(pk[pc] & 0xFFFF0000u)));
                        if (want_lse)
                            acc_exact[pc & 1] = f2_add(acc_exact[pc & 1], f2_pack(pe[2 * pc], pe[2 * pc + 1]));
                    }
                    {
                        const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
                        float a0, a1;
                        f2_unpack(a2, a0, a1);
                        l_t = a0 + a1;
                        f2_unpack(f2_add(acc_exact[0], acc_exact[1]), a0, a1);
                        le_t = a0 + a1;
                    }
                    if (with_max) break;
                    if (!__any_sync(0xFFFFFFFFu, !(l_t <= MAX_TILE_SUM))) break;
                }
                l_run = l_run * alpha + l_t;
                l_exact = l_exact * alpha + le_t;
                tmem_st64_nowait(tS, pk);
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
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.p_full);
                ++g;
            }
            if (!ok) break;

            // Epilogue: O / l, and the log-sum-exp. Reading O_s here, before this
            // warpgroup's next arrival on p_full, is what lets the next row's
            // first P V (which overwrites O_s) go ahead.
            if (nt > 0) {
                const bool w = mbar_wait_bounded(&B.o_full, rowc & 1, abort_flag, W_O_FULL, lim);
                ++rowc;
                if (!__all_sync(0xFFFFFFFFu, w)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            const bool have = nt > 0 && l_run > 0.f;
            const float inv_l = have ? 1.f / l_run : 0.f;
            uint32_t o[D];
            if (nt > 0) {
                if constexpr (D == 128) tmem_ld128(tO, o); else tmem_ld64(tO, o);
            } else {
#pragma unroll
                for (int e = 0; e < D; ++e) o[e] = 0u;
            }
            if (!prm.out_f32) {
                // bf16 O through the slot's staging tile and TMA stores, 64
                // channels at a time: each warp writes its 32 rows, the elected
                // thread stores the tile (rows past N or past the query block
                // are clipped by the store's box).
                const bool elected = (wq == 0 && lane == 0);
                uint8_t* stg = smem + L::OFF_STG + s * L::STG_BYTES;
                // This row of the staging tile: 128 bytes (64 channels), its 16-byte
                // chunks permuted by the 128-byte swizzle (chunk c at c ^ (row mod 8)).
                const uint32_t stg_row = smem_u32(stg) + (uint32_t)row * 128u;
                const uint32_t swz = (uint32_t)(row & 7);
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    if (npass > 0) {
                        // The previous store has read the tile: it may be rewritten.
                        if (elected) {
                            bulk_wait_group_read0();
                            mbar_arrive(&B.stg_free);
                        }
                        const bool w = mbar_wait_bounded(&B.stg_free, (npass - 1) & 1, abort_flag, W_STG, lim);
                        if (!__all_sync(0xFFFFFFFFu, w)) {
                            ok = false;
                            break;
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t* oc = o + 64 * h + 8 * c;
                        st_shared_v4(stg_row + (((uint32_t)c ^ swz) << 4),
                                     pack_bf16x2(__uint_as_float(oc[0]) * inv_l, __uint_as_float(oc[1]) * inv_l),
                                     pack_bf16x2(__uint_as_float(oc[2]) * inv_l, __uint_as_float(oc[3]) * inv_l),
                                     pack_bf16x2(__uint_as_float(oc[4]) * inv_l, __uint_as_float(oc[5]) * inv_l),
                                     pack_bf16x2(__uint_as_float(oc[6]) * inv_l, __uint_as_float(oc[7]) * inv_l));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&B.stg_full);
                    bool w = true;
                    if (elected) {
                        w = mbar_wait_bounded(&B.stg_full, npass & 1, abort_flag, W_STG, lim);
                        if (w) {
                            tma_store_3d(&tmO, stg, h * 64, qb * BQ, bh);
                            bulk_commit_group();
                        }
                    }
                    ++npass;
                    if (!__all_sync(0xFFFFFFFFu, w)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
            } else if (row_valid) {
                float4* out = reinterpret_cast<float4*>(static_cast<float*>(prm.O) + out_off);
#pragma unroll
                for (int e4 = 0; e4 < D / 4; ++e4)
                    out[e4] = make_float4(__uint_as_float(o[4 * e4 + 0]) * inv_l, __uint_as_float(o[4 * e4 + 1]) * inv_l,
                                          __uint_as_float(o[4 * e4 + 2]) * inv_l, __uint_as_float(o[4 * e4 + 3]) * inv_l);
            }
            if (want_lse && row_valid)
                prm.lse[(size_t)bh * prm.N + q_tok] = have ? (m_run + __log2f(l_exact)) * 0.69314718055994531f : -INFINITY;
        }
        // Every tile store has completed before the CTA (and its shared memory) ends.
        if (wq == 0 && lane == 0) bulk_wait_group0();
        tc_fence_before();
    }

    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace attn
}  // namespace sa
