// sa_lib.cu - the C ABI of libsparse_attn.so (declared in include/sparse_attn.h):
// argument validation, tensor-map encoding, kernel launches, and the device
// error record. The library is one translation unit: the kernels live in
// the included headers.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <cuda.h>
#include <cuda_runtime.h>

#include "sparse_attn.h"
#include "sparse_attn_testing.h"
#include "sa_ptx.cuh"
#include "sa_mask_kernels.cuh"
#include "sa_attn_kernel.cuh"
#include "sa_bwd_kernels.cuh"
#include "sa_fp8_kernels.cuh"
#include "sa_linear_kernels.cuh"
#include "sa_kmeans_kernels.cuh"

namespace {

thread_local std::string t_last_error;

sa_status fail(sa_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

sa_status ok() {
    t_last_error.clear();
    return SA_OK;
}

sa_status cuda_check(cudaError_t e, const char* what) {
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return SA_OK;
}

constexpr int MAX_NK = 8192;
constexpr unsigned long long WAIT_LIMIT_NS = 4000000000ull;  // 4 s per pipeline wait

struct Dims {
    int B, H, N, d, bq, bk, n_q, n_k, BH;
};

sa_status check_shape(const sa_shape* s, Dims& o) {
    if (!s) return fail(SA_ERR_INVALID_ARG, "shape is NULL");
    if (s->B <= 0 || s->H <= 0 || s->N <= 0 || s->d <= 0 || s->bq <= 0 || s->bk <= 0)
        return fail(SA_ERR_INVALID_ARG, "non-positive size in shape (B=%d H=%d N=%d d=%d bq=%d bk=%d)",
                    s->B, s->H, s->N, s->d, s->bq, s->bk);
    if (s->d != 64 && s->d != 128) return fail(SA_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", s->d);
    if (s->bq != 64 && s->bq != 128)
        return fail(SA_ERR_UNSUPPORTED, "bq=%d (supported: 64, 128)", s->bq);
    if (s->bk != 64) return fail(SA_ERR_UNSUPPORTED, "bk=%d (supported: 64)", s->bk);
    const long long BH = (long long)s->B * s->H;
    if (BH > 65535) return fail(SA_ERR_UNSUPPORTED, "B*H=%lld exceeds 65535", BH);
    o.B = s->B;
    o.H = s->H;
    o.N = s->N;
    o.d = s->d;
    o.bq = s->bq;
    o.bk = s->bk;
    o.BH = (int)BH;
    o.n_q = (s->N + s->bq - 1) / s->bq;
    o.n_k = (s->N + s->bk - 1) / s->bk;
    if (o.n_k > MAX_NK) return fail(SA_ERR_UNSUPPORTED, "n_k=%d exceeds %d", o.n_k, MAX_NK);
    return SA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sa_status check_kp(double k, double p) {
    if (!std::isfinite(k) || !std::isfinite(p) || k < 0.0 || k > 1.0 || p < 0.0 || p > 1.0)
        return fail(SA_ERR_INVALID_ARG, "k=%g p=%g: both must lie in [0, 1]", k, p);
    if (k == 0.0 && p == 0.0) return fail(SA_ERR_INVALID_ARG, "k = p = 0 keeps no block");
    return SA_OK;
}

// Top-k count: ceil(k * n_k) in double with a 1e-9 guard (k >= 1 keeps all).
int topk_count(double k, int n_k) {
    if (k >= 1.0) return n_k;
    double c = std::ceil(k * (double)n_k - 1e-9);
    if (c < 0.0) c = 0.0;
    if (c > (double)n_k) c = (double)n_k;
    return (int)c;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct Workspace {
    size_t qbar, kbar, logits, total;
    int ld;
};

Workspace workspace_layout(const Dims& g) {
    Workspace w;
    w.ld = (g.n_k + 3) & ~3;
    w.qbar = 0;
    w.kbar = round256((size_t)g.BH * g.n_q * g.d * sizeof(float));
    w.logits = w.kbar + round256((size_t)g.BH * g.n_k * g.d * sizeof(float));
    w.total = w.logits + round256((size_t)g.BH * g.n_q * w.ld * sizeof(float));
    return w;
}

// ---------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [BH, N, d] bf16 viewed as a 3-D tensor (d, N, BH); box = 64 channels x
// `rows` tokens x 1 head, 128-byte swizzle; out-of-range rows read as zero
// (and are not written by a store).
sa_status make_map(CUtensorMap* map, const void* base, const Dims& g, int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.BH};
    const cuuint64_t strides[2] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.N * g.d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return SA_OK;
}

// [BH, N, d] e4m3 codes (one byte each) viewed as (d, N, BH); box = 128
// channels (128 bytes) x `rows` tokens x 1 head, 128-byte swizzle.
sa_status make_map_u8(CUtensorMap* map, const void* base, const Dims& g, int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.BH};
    const cuuint64_t strides[2] = {(cuuint64_t)g.d, (cuuint64_t)g.N * g.d};
    const cuuint32_t box[3] = {128, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed (CUresult %d)", (int)r);
    return SA_OK;
}

// ------------------------------------------------------------ launches
template <int D>
sa_status launch_pool_score(const Dims& g, const void* Q, const void* K, const Workspace& w,
                            uint8_t* ws, cudaStream_t st) {
    float* qbar = reinterpret_cast<float*>(ws + w.qbar);
    float* kbar = reinterpret_cast<float*>(ws + w.kbar);
    float* logits = reinterpret_cast<float*>(ws + w.logits);
    dim3 pg(g.n_q + g.n_k, g.BH);
    sa::mask::pool_kernel<D><<<pg, sa::mask::POOL_THREADS, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(Q), reinterpret_cast<const __nv_bfloat16*>(K), qbar,
        kbar, g.N, g.bq, g.bk, g.n_q, g.n_k);
    sa_status s = cuda_check(cudaGetLastError(), "pool_kernel launch");
    if (s != SA_OK) return s;
    dim3 sg((g.n_k + sa::mask::SC_TJ - 1) / sa::mask::SC_TJ, (g.n_q + sa::mask::SC_TI - 1) / sa::mask::SC_TI,
            g.BH);
    const float scale = (float)(1.0 / std::sqrt((double)D));
    sa::mask::score_kernel<D><<<sg, sa::mask::SC_THREADS, 0, st>>>(qbar, kbar, logits, w.ld, g.n_q,
                                                                   g.n_k, scale);
    return cuda_check(cudaGetLastError(), "score_kernel launch");
}

template <bool FROM_LOGITS>
sa_status launch_select(const Dims& g, const float* in, int ld_in, double k, double p, int32_t* cnt,
                        int32_t* idx, uint8_t* mask, float* P_out, cudaStream_t st) {
    const int rows = g.BH * g.n_q;
    const int wpc = sa::mask::select_warps_per_cta(g.n_k);
    const size_t smem = (size_t)wpc * sa::mask::select_row_bytes(g.n_k);
    auto kern = sa::mask::select_kernel<FROM_LOGITS>;
    // Set on every call: the attribute is per device.
    sa_status s = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  sa::mask::SEL_SMEM_BUDGET),
                             "select_kernel shared-memory attribute");
    if (s != SA_OK) return s;
    const int grid = (rows + wpc - 1) / wpc;
    kern<<<grid, wpc * 32, smem, st>>>(in, ld_in, rows, g.n_k, topk_count(k, g.n_k), p, cnt, idx, mask,
                                       P_out);
    return cuda_check(cudaGetLastError(), "select_kernel launch");
}

// Multiprocessor count of the current device (cached per device).
int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Knobs of the failure-detection test hook; normal launches use the defaults.
struct AttnTestKnobs {
    unsigned long long wait_limit_ns = WAIT_LIMIT_NS;
    int withhold_first_k = 0;
};

// The FP8 path's per-block scales (null on the bf16 path).
struct Fp8Scales {
    const float* q = nullptr;
    const float* k = nullptr;
};

// The single-launch path's extra arguments (the mask phases).
struct FusedArgs {
    float* qbar = nullptr;
    float* kbar = nullptr;
    unsigned int* grid_ctr = nullptr;
    int kc = 0;
    double p = 0.0;
};

template <int D, int BQ, bool FP8 = false, bool FUSED = false>
sa_status launch_attn_t(const Dims& g, const void* Q, const void* K, const void* V, const int32_t* cnt,
                        const int32_t* idx, void* O, bool out_f32, float* lse, bool dense,
                        cudaStream_t st, const AttnTestKnobs& knobs, const Fp8Scales& sc = Fp8Scales(),
                        const FusedArgs& fz = FusedArgs()) {
    using L = sa::attn::Layout<D, FP8>;
    CUtensorMap mq, mk, mv, mo;
    sa_status s;
    if (FP8) {
        if ((s = make_map_u8(&mq, Q, g, sa::attn::MROWS)) != SA_OK) return s;
        if ((s = make_map_u8(&mk, K, g, sa::attn::BK)) != SA_OK) return s;
    } else {
        if ((s = make_map(&mq, Q, g, sa::attn::MROWS)) != SA_OK) return s;
        if ((s = make_map(&mk, K, g, sa::attn::BK)) != SA_OK) return s;
    }
    if ((s = make_map(&mv, V, g, sa::attn::BK)) != SA_OK) return s;
    // bf16 O is written by tile stores of 64 channels x one query block; the
    // fp32 output is written directly (the map is then unused).
    if (out_f32) mo = mq;
    else if ((s = make_map(&mo, O, g, BQ)) != SA_OK) return s;
    auto kern = sa::attn::sparse_attn_fwd_kernel<D, BQ, FP8, FUSED>;
    if ((s = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::DYN_BYTES),
                        "sparse_attn_fwd_kernel shared-memory attribute")) != SA_OK)
        return s;
    // The kernel moves registers between its warpgroups (setmaxnreg); the
    // split adds up only for the launch register count it was written for.
    cudaFuncAttributes fa;
    if ((s = cuda_check(cudaFuncGetAttributes(&fa, kern), "sparse_attn_fwd_kernel attributes")) != SA_OK) return s;
    if (fa.numRegs != sa::attn::LAUNCH_REGS)
        return fail(SA_ERR_UNSUPPORTED, "sparse_attn_fwd_kernel was built with %d registers per thread, not %d",
                    fa.numRegs, sa::attn::LAUNCH_REGS);
    sa::attn::Params prm;
    prm.cnt = cnt;
    prm.idx = idx;
    prm.O = O;
    prm.lse = lse;
    prm.N = g.N;
    prm.n_q = g.n_q;
    prm.n_k = g.n_k;
    prm.rows = g.BH * g.n_q;
    prm.dense = dense ? 1 : 0;
    prm.out_f32 = out_f32 ? 1 : 0;
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    prm.wait_limit_ns = knobs.wait_limit_ns;
    prm.withhold_first_k = knobs.withhold_first_k;
    prm.q_scale = sc.q;
    prm.k_scale = sc.k;
    prm.q_in = Q;
    prm.k_in = K;
    prm.qbar = fz.qbar;
    prm.kbar = fz.kbar;
    prm.grid_ctr = fz.grid_ctr;
    prm.cnt_w = const_cast<int32_t*>(cnt);
    prm.idx_w = const_cast<int32_t*>(idx);
    prm.BH = g.BH;
    prm.bq = g.bq;
    prm.kc = fz.kc;
    prm.p = fz.p;
    prm.score_scale = (float)(1.0 / std::sqrt((double)D));
    // Persistent: one CTA per multiprocessor (fewer when there are fewer row pairs).
    const int pairs = (prm.rows + sa::attn::NSLOT - 1) / sa::attn::NSLOT;
    const int grid = pairs < sm_count() ? pairs : sm_count();
    if constexpr (FUSED) {
        // Cooperative launch: the grid barriers need every CTA resident at
        // once, which the launch guarantees (or refuses).
        if ((s = cuda_check(cudaMemsetAsync(fz.grid_ctr, 0, sizeof(unsigned int), st), "zero the grid counter")) !=
            SA_OK)
            return s;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(sa::attn::NUM_THREADS);
        cfg.dynamicSmemBytes = L::DYN_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cuda_check(cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, prm), "single-launch kernel launch");
    }
    kern<<<grid, sa::attn::NUM_THREADS, L::DYN_BYTES, st>>>(mq, mk, mv, mo, prm);
    return cuda_check(cudaGetLastError(), "sparse_attn_fwd_kernel launch");
}

sa_status launch_fwd(const Dims& g, const void* Q, const void* K, const void* V, const int32_t* cnt,
                     const int32_t* idx, void* O, bool out_f32, float* lse, bool dense,
                     cudaStream_t st, const AttnTestKnobs& knobs = AttnTestKnobs()) {
    if (g.d == 128 && g.bq == 128)
        return launch_attn_t<128, 128>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st, knobs);
    if (g.d == 128 && g.bq == 64)
        return launch_attn_t<128, 64>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st, knobs);
    if (g.d == 64 && g.bq == 128)
        return launch_attn_t<64, 128>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st, knobs);
    return launch_attn_t<64, 64>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st, knobs);
}

sa_status check_out_dtype(int o_dtype) {
    if (o_dtype != SA_BF16 && o_dtype != SA_F32)
        return fail(SA_ERR_INVALID_ARG, "o_dtype=%d (SA_BF16=0 or SA_F32=1)", o_dtype);
    return SA_OK;
}

sa_status check_fwd_args(const sa_shape* shape, const void* Q, const void* K, const void* V,
                         const int32_t* cnt, const int32_t* idx, void* O, int o_dtype,
                         const float* lse_or_null, Dims& g) {
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_out_dtype(o_dtype)) != SA_OK) return s;
    if (!Q || !K || !V || !cnt || !idx || !O)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, V, cnt, idx, O");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(cnt) || !aligned16(idx) ||
        !aligned16(O) || (lse_or_null && !aligned16(lse_or_null)))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    return SA_OK;
}

// ------------------------------------------------------------ backward
struct BwdWorkspace {
    size_t lsed, bitmap, ucnt, uidx, total;
    int nw, n_kp;
};

BwdWorkspace bwd_layout(const Dims& g) {
    BwdWorkspace w;
    w.nw = (g.n_k + 31) / 32;
    w.n_kp = (g.n_k + 1) / 2;
    w.lsed = 0;
    w.bitmap = round256((size_t)g.BH * g.n_q * g.bq * sizeof(float2));
    w.ucnt = w.bitmap + round256((size_t)g.BH * g.n_q * w.nw * sizeof(uint32_t));
    w.uidx = w.ucnt + round256((size_t)g.BH * w.n_kp * sizeof(int32_t));
    w.total = w.uidx + round256((size_t)g.BH * w.n_kp * g.n_q * sizeof(int32_t));
    return w;
}

template <typename KernelT>
sa_status prepare_tc_kernel(KernelT kern, int dyn_bytes, const char* name) {
    sa_status s;
    if ((s = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_bytes),
                        name)) != SA_OK)
        return s;
    // The kernel moves registers between its warpgroups (setmaxnreg); the
    // split adds up only for the launch register count it was written for.
    cudaFuncAttributes fa;
    if ((s = cuda_check(cudaFuncGetAttributes(&fa, kern), name)) != SA_OK) return s;
    if (fa.numRegs != sa::bwd::LAUNCH_REGS)
        return fail(SA_ERR_UNSUPPORTED, "%s was built with %d registers per thread, not %d", name, fa.numRegs,
                    sa::bwd::LAUNCH_REGS);
    return SA_OK;
}

template <int D, int BQ>
sa_status launch_bwd_t(const Dims& g, const void* Q, const void* K, const void* V, const void* O, const void* dO,
                       const float* lse, const int32_t* cnt, const int32_t* idx, void* dQ, void* dK, void* dV,
                       bool out_f32, uint8_t* ws, cudaStream_t st) {
    const BwdWorkspace w = bwd_layout(g);
    float2* lsed = reinterpret_cast<float2*>(ws + w.lsed);
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(ws + w.bitmap);
    int32_t* ucnt = reinterpret_cast<int32_t*>(ws + w.ucnt);
    int32_t* uidx = reinterpret_cast<int32_t*>(ws + w.uidx);
    sa_status s;
    sa::bwd::bwd_rows_kernel<D><<<dim3(g.n_q, g.BH), 128, w.nw * sizeof(uint32_t), st>>>(
        reinterpret_cast<const __nv_bfloat16*>(O), reinterpret_cast<const __nv_bfloat16*>(dO), lse, cnt, idx, lsed,
        bitmap, g.N, g.bq, g.n_q, g.n_k, w.nw);
    if ((s = cuda_check(cudaGetLastError(), "bwd_rows_kernel launch")) != SA_OK) return s;
    sa::bwd::bwd_transpose_kernel<<<dim3((w.nw + sa::bwd::TR_WARPS - 1) / sa::bwd::TR_WARPS, g.BH),
                                    sa::bwd::TR_WARPS * 32, 0, st>>>(bitmap, ucnt, uidx, g.n_q, w.nw, w.n_kp);
    if ((s = cuda_check(cudaGetLastError(), "bwd_transpose_kernel launch")) != SA_OK) return s;

    CUtensorMap mq128, mdo128, mqb, mdob, mk, mv;
    if ((s = make_map(&mq128, Q, g, sa::bwd::MROWS)) != SA_OK || (s = make_map(&mdo128, dO, g, sa::bwd::MROWS)) != SA_OK ||
        (s = make_map(&mqb, Q, g, BQ)) != SA_OK || (s = make_map(&mdob, dO, g, BQ)) != SA_OK ||
        (s = make_map(&mk, K, g, sa::bwd::BK)) != SA_OK || (s = make_map(&mv, V, g, sa::bwd::BK)) != SA_OK)
        return s;
    sa::bwd::Params prm;
    prm.lsed = lsed;
    prm.N = g.N;
    prm.n_q = g.n_q;
    prm.n_k = g.n_k;
    prm.n_kp = w.n_kp;
    prm.out_f32 = out_f32 ? 1 : 0;
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    prm.scale = (float)(1.0 / std::sqrt((double)D));
    prm.wait_limit_ns = WAIT_LIMIT_NS;

    auto kdq = sa::bwd::bwd_dq_kernel<D, BQ>;
    constexpr int DQ_BYTES = sa::bwd::DQLayout<D, BQ>::DYN_BYTES;
    if ((s = prepare_tc_kernel(kdq, DQ_BYTES, "bwd_dq_kernel")) != SA_OK) return s;
    sa::bwd::Params pq = prm;
    pq.cnt = cnt;
    pq.idx = idx;
    pq.out0 = dQ;
    pq.out1 = nullptr;
    pq.items = g.BH * g.n_q;
    const int gq = pq.items < sm_count() ? pq.items : sm_count();
    kdq<<<gq, sa::bwd::NUM_THREADS, DQ_BYTES, st>>>(mq128, mk, mv, mdo128, pq);
    if ((s = cuda_check(cudaGetLastError(), "bwd_dq_kernel launch")) != SA_OK) return s;

    auto kkv = sa::bwd::bwd_dkdv_kernel<D, BQ>;
    constexpr int KV_BYTES = sa::bwd::KVLayout<D, BQ>::DYN_BYTES;
    if ((s = prepare_tc_kernel(kkv, KV_BYTES, "bwd_dkdv_kernel")) != SA_OK) return s;
    sa::bwd::Params pk = prm;
    pk.cnt = ucnt;
    pk.idx = uidx;
    pk.out0 = dV;
    pk.out1 = dK;
    pk.items = g.BH * w.n_kp;
    const int gk = pk.items < sm_count() ? pk.items : sm_count();
    kkv<<<gk, sa::bwd::NUM_THREADS, KV_BYTES, st>>>(mqb, mk, mv, mdob, pk);
    return cuda_check(cudaGetLastError(), "bwd_dkdv_kernel launch");
}

sa_status launch_bwd(const Dims& g, const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     const float* lse, const int32_t* cnt, const int32_t* idx, void* dQ, void* dK, void* dV,
                     bool out_f32, uint8_t* ws, cudaStream_t st) {
    if (g.d == 128 && g.bq == 128)
        return launch_bwd_t<128, 128>(g, Q, K, V, O, dO, lse, cnt, idx, dQ, dK, dV, out_f32, ws, st);
    if (g.d == 128 && g.bq == 64)
        return launch_bwd_t<128, 64>(g, Q, K, V, O, dO, lse, cnt, idx, dQ, dK, dV, out_f32, ws, st);
    if (g.d == 64 && g.bq == 128)
        return launch_bwd_t<64, 128>(g, Q, K, V, O, dO, lse, cnt, idx, dQ, dK, dV, out_f32, ws, st);
    return launch_bwd_t<64, 64>(g, Q, K, V, O, dO, lse, cnt, idx, dQ, dK, dV, out_f32, ws, st);
}

// ------------------------------------------------- sparse + linear (SLA2)
struct LinWorkspace {
    size_t pq, pk, zpart, hpart, hhi, hlo, z, total;
    int n_b, splits, n_chunks;
};

LinWorkspace lin_layout(const Dims& g) {
    LinWorkspace w;
    w.n_b = (g.N + 63) / 64;
    w.n_chunks = (g.N + sa::lin::LS_CHUNK - 1) / sa::lin::LS_CHUNK;
    int sp = (sm_count() + g.BH - 1) / g.BH;   // about one wave of state CTAs
    if (sp > w.n_chunks) sp = w.n_chunks;
    w.splits = sp < 1 ? 1 : sp;
    const size_t tok = (size_t)g.BH * g.N * g.d;
    w.pq = 0;
    w.pk = w.pq + round256(tok * 2);
    w.zpart = w.pk + round256(tok * 2);
    w.hpart = w.zpart + round256((size_t)g.BH * w.n_b * g.d * 4);
    w.hhi = w.hpart + round256((size_t)g.BH * w.splits * g.d * g.d * 4);
    w.hlo = w.hhi + round256((size_t)g.BH * g.d * g.d * 2);
    w.z = w.hlo + round256((size_t)g.BH * g.d * g.d * 2);
    w.total = w.z + round256((size_t)g.BH * g.d * 4);
    return w;
}

template <int BQ>
sa_status launch_sparse_linear(const Dims& g, const void* Q, const void* K, const void* V, const int32_t* cnt,
                               const int32_t* idx, const void* Os, const float* alpha, void* O, bool out_f32,
                               uint8_t* ws, cudaStream_t st) {
    constexpr int D = 128;
    const LinWorkspace w = lin_layout(g);
    auto* pQ = reinterpret_cast<__nv_bfloat16*>(ws + w.pq);
    auto* pK = reinterpret_cast<__nv_bfloat16*>(ws + w.pk);
    float* zpart = reinterpret_cast<float*>(ws + w.zpart);
    float* hpart = reinterpret_cast<float*>(ws + w.hpart);
    auto* Hhi = reinterpret_cast<__nv_bfloat16*>(ws + w.hhi);
    auto* Hlo = reinterpret_cast<__nv_bfloat16*>(ws + w.hlo);
    float* z = reinterpret_cast<float*>(ws + w.z);
    sa_status s;
    sa::lin::phi_kernel<D><<<dim3(2 * w.n_b, g.BH), 128, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(Q), reinterpret_cast<const __nv_bfloat16*>(K), pQ, pK, zpart, g.N, w.n_b);
    if ((s = cuda_check(cudaGetLastError(), "phi_kernel launch")) != SA_OK) return s;

    CUtensorMap m_pk128, m_v128;
    if ((s = make_map(&m_pk128, pK, g, sa::lin::LS_CHUNK)) != SA_OK || (s = make_map(&m_v128, V, g, sa::lin::LS_CHUNK)) != SA_OK)
        return s;
    using LSL = sa::lin::LSLayout<D>;
    auto kls = sa::lin::lin_state_kernel<D>;
    if ((s = cuda_check(cudaFuncSetAttribute(kls, cudaFuncAttributeMaxDynamicSharedMemorySize, LSL::DYN_BYTES),
                        "lin_state_kernel shared-memory attribute")) != SA_OK)
        return s;
    kls<<<dim3(g.BH, w.splits), sa::lin::LS_THREADS, LSL::DYN_BYTES, st>>>(m_pk128, m_v128, hpart, w.n_chunks, w.splits,
                                                                          WAIT_LIMIT_NS);
    if ((s = cuda_check(cudaGetLastError(), "lin_state_kernel launch")) != SA_OK) return s;
    sa::lin::lin_finalize_kernel<D><<<g.BH, D, 0, st>>>(hpart, zpart, Hhi, Hlo, z, w.splits, w.n_b);
    if ((s = cuda_check(cudaGetLastError(), "lin_finalize_kernel launch")) != SA_OK) return s;

    CUtensorMap m_pq, m_pk, m_v, m_hhi, m_hlo;
    Dims gh = g;
    gh.N = D;   // H, viewed as D rows of D channels per head
    if ((s = make_map(&m_pq, pQ, g, sa::lin::SL_MROWS)) != SA_OK || (s = make_map(&m_pk, pK, g, sa::lin::SL_BK)) != SA_OK ||
        (s = make_map(&m_v, V, g, sa::lin::SL_BK)) != SA_OK || (s = make_map(&m_hhi, Hhi, gh, 128)) != SA_OK ||
        (s = make_map(&m_hlo, Hlo, gh, 128)) != SA_OK)
        return s;
    using SLL = sa::lin::SLLayout<D>;
    auto ksl = sa::lin::sparse_linear_kernel<D, BQ>;
    if ((s = cuda_check(cudaFuncSetAttribute(ksl, cudaFuncAttributeMaxDynamicSharedMemorySize, SLL::DYN_BYTES),
                        "sparse_linear_kernel shared-memory attribute")) != SA_OK)
        return s;
    sa::lin::SLParams prm;
    prm.cnt = cnt;
    prm.idx = idx;
    prm.pQ = pQ;
    prm.z = z;
    prm.Os = Os;
    prm.alpha = alpha;
    prm.O = O;
    prm.N = g.N;
    prm.n_q = g.n_q;
    prm.n_k = g.n_k;
    prm.rows = g.BH * g.n_q;
    prm.out_f32 = out_f32 ? 1 : 0;
    prm.wait_limit_ns = WAIT_LIMIT_NS;
    const int grid = prm.rows < sm_count() ? prm.rows : sm_count();
    ksl<<<grid, sa::lin::SL_THREADS, SLL::DYN_BYTES, st>>>(m_pq, m_pk, m_v, m_hhi, m_hlo, prm);
    return cuda_check(cudaGetLastError(), "sparse_linear_kernel launch");
}

// ------------------------------------------------- single-launch path
// Workspace: the block means (fp32, as the mask's) and the grid counter.
struct FusedLayout {
    size_t qbar, kbar, ctr, total;
};

FusedLayout fused_layout(const Dims& g) {
    FusedLayout w;
    w.qbar = 0;
    w.kbar = round256((size_t)g.BH * g.n_q * g.d * sizeof(float));
    w.ctr = w.kbar + round256((size_t)g.BH * g.n_k * g.d * sizeof(float));
    w.total = w.ctr + 256;
    return w;
}

// The selection phase keeps a tile of rows' logits and masses in the
// attention kernel's shared memory (below its control block).
sa_status check_fused_shape(const Dims& g) {
    const size_t room = g.d == 128 ? (size_t)sa::attn::Layout<128>::OFF_CTRL : (size_t)sa::attn::Layout<64>::OFF_CTRL;
    const size_t need = sa::mask::fused_select_smem(g.d, g.n_k);
    if (need > room)
        return fail(SA_ERR_UNSUPPORTED, "single-launch path: n_k=%d needs %zu bytes of shared memory for its "
                    "selection phase, %zu available (use sparse_attn_mask + sparse_attn_fwd)", g.n_k, need, room);
    return SA_OK;
}

// ------------------------------------------- semantic-aware permutation
constexpr int KM_MAX_C = 8192;
constexpr int KM_MAX_ITERS = 100;

sa_status check_kmeans(const sa_shape* shape, int C, int iters, Dims& g) {
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if (C < 1 || C > g.N || C > KM_MAX_C)
        return fail(SA_ERR_INVALID_ARG, "C=%d clusters: need 1 <= C <= min(N=%d, %d)", C, g.N, KM_MAX_C);
    if (iters < 0 || iters > KM_MAX_ITERS) return fail(SA_ERR_INVALID_ARG, "iters=%d outside [0, %d]", iters, KM_MAX_ITERS);
    return SA_OK;
}

template <int D>
sa_status launch_kmeans(const Dims& g, const void* X, int C, int iters, const float* init, int32_t* ids,
                        int32_t* perm, float* M, int32_t* off, cudaStream_t st) {
    auto* x = reinterpret_cast<const __nv_bfloat16*>(X);
    sa_status s;
    if (init) {
        // Cached centroids (the output buffer itself when the caller updates them in place).
        if (init != M &&
            (s = cuda_check(cudaMemcpyAsync(M, init, (size_t)g.BH * C * D * sizeof(float), cudaMemcpyDeviceToDevice, st),
                            "copy the initial centroids")) != SA_OK)
            return s;
    } else {
        sa::km::km_init_kernel<D><<<dim3(C, g.BH), D, 0, st>>>(x, M, g.N, C);
        if ((s = cuda_check(cudaGetLastError(), "km_init_kernel launch")) != SA_OK) return s;
    }
    const dim3 ag((g.N + sa::km::AS_THREADS - 1) / sa::km::AS_THREADS, g.BH);
    constexpr size_t SORT_SMEM_BUDGET = 200 * 1024;
    const int sw = sa::km::km_sort_warps(C, SORT_SMEM_BUDGET);
    const size_t sort_smem = (size_t)(sw + 1) * C * sizeof(int32_t);
    if ((s = cuda_check(cudaFuncSetAttribute(sa::km::km_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SORT_SMEM_BUDGET),
                        "km_sort_kernel shared-memory attribute")) != SA_OK)
        return s;
    for (int it = 0; it <= iters; ++it) {
        sa::km::km_assign_kernel<D><<<ag, sa::km::AS_THREADS, 0, st>>>(x, M, ids, g.N, C);
        if ((s = cuda_check(cudaGetLastError(), "km_assign_kernel launch")) != SA_OK) return s;
        sa::km::km_sort_kernel<<<g.BH, 32 * sw, sort_smem, st>>>(ids, perm, off, g.N, C);
        if ((s = cuda_check(cudaGetLastError(), "km_sort_kernel launch")) != SA_OK) return s;
        if (it == iters) break;   // the final assignment is not followed by an update
        sa::km::km_update_kernel<D><<<dim3(C, g.BH), D, 0, st>>>(x, perm, off, M, g.N, C);
        if ((s = cuda_check(cudaGetLastError(), "km_update_kernel launch")) != SA_OK) return s;
    }
    return SA_OK;
}

}  // namespace

extern "C" {

size_t sparse_attn_fused_workspace_bytes(const sa_shape* shape) {
    Dims g;
    if (check_shape(shape, g) != SA_OK || check_fused_shape(g) != SA_OK) return 0;
    return fused_layout(g).total;
}

sa_status sparse_attn_fused(const sa_shape* shape, const void* Q, const void* K, const void* V, double k, double p,
                            int32_t* cnt, int32_t* idx, void* O, int o_dtype, float* lse_or_null, void* workspace,
                            size_t workspace_bytes, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_fwd_args(shape, Q, K, V, cnt, idx, O, o_dtype, lse_or_null, g)) != SA_OK) return s;
    if ((s = check_kp(k, p)) != SA_OK) return s;
    if ((s = check_fused_shape(g)) != SA_OK) return s;
    if (!workspace) return fail(SA_ERR_INVALID_ARG, "NULL workspace");
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(SA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    const FusedLayout w = fused_layout(g);
    if (workspace_bytes < w.total)
        return fail(SA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, w.total);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    FusedArgs fa;
    fa.qbar = reinterpret_cast<float*>(ws + w.qbar);
    fa.kbar = reinterpret_cast<float*>(ws + w.kbar);
    fa.grid_ctr = reinterpret_cast<unsigned int*>(ws + w.ctr);
    fa.kc = topk_count(k, g.n_k);
    fa.p = p;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool f32 = o_dtype == SA_F32;
    const AttnTestKnobs kn;
    if (g.d == 128 && g.bq == 128)
        s = launch_attn_t<128, 128, false, true>(g, Q, K, V, cnt, idx, O, f32, lse_or_null, false, st, kn, {}, fa);
    else if (g.d == 128)
        s = launch_attn_t<128, 64, false, true>(g, Q, K, V, cnt, idx, O, f32, lse_or_null, false, st, kn, {}, fa);
    else if (g.bq == 128)
        s = launch_attn_t<64, 128, false, true>(g, Q, K, V, cnt, idx, O, f32, lse_or_null, false, st, kn, {}, fa);
    else
        s = launch_attn_t<64, 64, false, true>(g, Q, K, V, cnt, idx, O, f32, lse_or_null, false, st, kn, {}, fa);
    if (s != SA_OK) return s;
    return ok();
}

size_t sparse_attn_kmeans_workspace_bytes(const sa_shape* shape, int C) {
    Dims g;
    if (check_kmeans(shape, C, 0, g) != SA_OK) return 0;
    return round256((size_t)g.BH * (C + 1) * sizeof(int32_t));
}

sa_status sparse_attn_kmeans_permutation(const sa_shape* shape, const void* X, int C, int iters,
                                         const float* init_or_null, int32_t* ids, int32_t* perm, float* centroids,
                                         void* workspace, size_t workspace_bytes, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_kmeans(shape, C, iters, g)) != SA_OK) return s;
    if (!X || !ids || !perm || !centroids || !workspace)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among X, ids, perm, centroids, workspace");
    if (!aligned16(X) || !aligned16(ids) || !aligned16(perm) || !aligned16(centroids) ||
        (init_or_null && !aligned16(init_or_null)) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required; 256 for workspace)");
    const size_t need = round256((size_t)g.BH * (C + 1) * sizeof(int32_t));
    if (workspace_bytes < need) return fail(SA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t* off = reinterpret_cast<int32_t*>(workspace);
    s = (g.d == 128) ? launch_kmeans<128>(g, X, C, iters, init_or_null, ids, perm, centroids, off, st)
                     : launch_kmeans<64>(g, X, C, iters, init_or_null, ids, perm, centroids, off, st);
    if (s != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_permute_rows(const sa_shape* shape, const void* X, const int32_t* perm, void* Y, int dtype,
                                   int inverse, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_out_dtype(dtype)) != SA_OK) return s;
    if (!X || !perm || !Y) return fail(SA_ERR_INVALID_ARG, "NULL pointer among X, perm, Y");
    if (X == Y) return fail(SA_ERR_INVALID_ARG, "X and Y must not be the same buffer");
    if (!aligned16(X) || !aligned16(perm) || !aligned16(Y))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto* x = reinterpret_cast<const uint8_t*>(X);
    auto* y = reinterpret_cast<uint8_t*>(Y);
    const int row_bytes = g.d * (dtype == SA_F32 ? 4 : 2);
    auto grid = [&](int rows_per_cta) { return dim3((g.N + rows_per_cta - 1) / rows_per_cta, g.BH); };
    const int inv = inverse ? 1 : 0;
    if (row_bytes == 128)
        sa::km::permute_rows_kernel<128><<<grid(sa::km::PermuteShape<128>::ROWS_PER_CTA), 256, 0, st>>>(x, perm, y, g.N, inv);
    else if (row_bytes == 256)
        sa::km::permute_rows_kernel<256><<<grid(sa::km::PermuteShape<256>::ROWS_PER_CTA), 256, 0, st>>>(x, perm, y, g.N, inv);
    else
        sa::km::permute_rows_kernel<512><<<grid(sa::km::PermuteShape<512>::ROWS_PER_CTA), 256, 0, st>>>(x, perm, y, g.N, inv);
    if ((s = cuda_check(cudaGetLastError(), "permute_rows_kernel launch")) != SA_OK) return s;
    return ok();
}

size_t sparse_attn_sparse_linear_workspace_bytes(const sa_shape* shape) {
    Dims g;
    if (check_shape(shape, g) != SA_OK || g.d != 128) return 0;
    return lin_layout(g).total;
}

sa_status sparse_attn_sparse_linear(const sa_shape* shape, const void* Q, const void* K, const void* V,
                                    const int32_t* cnt, const int32_t* idx, const void* O_s, const float* alpha,
                                    void* O, int o_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_fwd_args(shape, Q, K, V, cnt, idx, O, o_dtype, nullptr, g)) != SA_OK) return s;
    if (g.d != 128) return fail(SA_ERR_UNSUPPORTED, "d=%d: the sparse + linear path supports d = 128", g.d);
    if (!O_s || !alpha || !workspace) return fail(SA_ERR_INVALID_ARG, "NULL pointer among O_s, alpha, workspace");
    if (!aligned16(O_s) || !aligned16(alpha) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required; 256 for workspace)");
    const size_t need = lin_layout(g).total;
    if (workspace_bytes < need)
        return fail(SA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    const bool f32 = o_dtype == SA_F32;
    s = (g.bq == 128) ? launch_sparse_linear<128>(g, Q, K, V, cnt, idx, O_s, alpha, O, f32, ws, st)
                      : launch_sparse_linear<64>(g, Q, K, V, cnt, idx, O_s, alpha, O, f32, ws, st);
    if (s != SA_OK) return s;
    return ok();
}

size_t sparse_attn_bwd_workspace_bytes(const sa_shape* shape) {
    Dims g;
    if (check_shape(shape, g) != SA_OK) return 0;
    return bwd_layout(g).total;
}

sa_status sparse_attn_bwd(const sa_shape* shape, const void* Q, const void* K, const void* V, const void* O,
                          const void* dO, const float* lse, const int32_t* cnt, const int32_t* idx, void* dQ,
                          void* dK, void* dV, int g_dtype, void* workspace, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_out_dtype(g_dtype)) != SA_OK) return s;
    if (!Q || !K || !V || !O || !dO || !lse || !cnt || !idx || !dQ || !dK || !dV || !workspace)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, V, O, dO, lse, cnt, idx, dQ, dK, dV, workspace");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(lse) ||
        !aligned16(cnt) || !aligned16(idx) || !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required; 256 for workspace)");
    s = launch_bwd(g, Q, K, V, O, dO, lse, cnt, idx, dQ, dK, dV, g_dtype == SA_F32,
                   reinterpret_cast<uint8_t*>(workspace), reinterpret_cast<cudaStream_t>(stream));
    if (s != SA_OK) return s;
    return ok();
}

size_t sparse_attn_mask_workspace_bytes(const sa_shape* shape) {
    Dims g;
    if (check_shape(shape, g) != SA_OK) return 0;
    return workspace_layout(g).total;
}

sa_status sparse_attn_mask(const sa_shape* shape, const void* Q, const void* K, double k, double p,
                           int32_t* cnt, int32_t* idx, uint8_t* mask_or_null, float* P_out_or_null,
                           void* workspace, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_kp(k, p)) != SA_OK) return s;
    if (!Q || !K || !cnt || !idx || !workspace)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, cnt, idx, workspace");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(cnt) || !aligned16(idx) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        (mask_or_null && !aligned16(mask_or_null)) || (P_out_or_null && !aligned16(P_out_or_null)))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required; 256 for workspace)");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const Workspace w = workspace_layout(g);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    s = (g.d == 128) ? launch_pool_score<128>(g, Q, K, w, ws, st) : launch_pool_score<64>(g, Q, K, w, ws, st);
    if (s != SA_OK) return s;
    s = launch_select<true>(g, reinterpret_cast<const float*>(ws + w.logits), w.ld, k, p, cnt, idx,
                            mask_or_null, P_out_or_null, st);
    if (s != SA_OK) return s;
    return ok();
}

}  // extern "C"

// ------------------------------------------------- allocation-free mask
// The scratch of sparse_attn_mask_noalloc: a fixed device array, one per
// device that loads this library, alive until the process exits. In host
// code `g_noalloc_scratch` is only a stand-in for the symbol, never a device
// address: kernels get the address that cudaGetSymbolAddress returns for the
// current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SPARSE_ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[NOALLOC_MAX_DEVICES] = {};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
sa_status noalloc_scratch(void** out) {
    int dev = -1;
    sa_status s = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
    if (s != SA_OK) return s;
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES)
        return fail(SA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, NOALLOC_MAX_DEVICES);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        s = cuda_check(cudaGetSymbolAddress(&ptr, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
        if (s != SA_OK) return s;
        if (!ptr) return fail(SA_ERR_CUDA, "scratch array has no device address");
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return SA_OK;
}

}  // namespace

extern "C" {

sa_status sparse_attn_mask_noalloc(const sa_shape* shape, const void* Q, const void* K, double k,
                                   double p, int32_t* cnt, int32_t* idx, uint8_t* mask_or_null,
                                   float* P_out_or_null, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    const size_t need = workspace_layout(g).total;
    if (need > (size_t)SPARSE_ATTN_NOALLOC_SCRATCH_BYTES)
        return fail(SA_ERR_UNSUPPORTED,
                    "workspace of %zu bytes exceeds the %u-byte scratch of sparse_attn_mask_noalloc; "
                    "use sparse_attn_mask with a caller-provided workspace",
                    need, (unsigned)SPARSE_ATTN_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != SA_OK) return s;
    return sparse_attn_mask(shape, Q, K, k, p, cnt, idx, mask_or_null, P_out_or_null, scratch, stream);
}

sa_status sparse_attn_select(const sa_shape* shape, const float* P, double k, double p, int32_t* cnt,
                             int32_t* idx, uint8_t* mask_or_null, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_kp(k, p)) != SA_OK) return s;
    if (!P || !cnt || !idx) return fail(SA_ERR_INVALID_ARG, "NULL pointer among P, cnt, idx");
    if (!aligned16(P) || !aligned16(cnt) || !aligned16(idx) || (mask_or_null && !aligned16(mask_or_null)))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    s = launch_select<false>(g, P, g.n_k, k, p, cnt, idx, mask_or_null, nullptr,
                             reinterpret_cast<cudaStream_t>(stream));
    if (s != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_fwd(const sa_shape* shape, const void* Q, const void* K, const void* V,
                          const int32_t* cnt, const int32_t* idx, void* O, int o_dtype,
                          float* lse_or_null, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_fwd_args(shape, Q, K, V, cnt, idx, O, o_dtype, lse_or_null, g)) != SA_OK) return s;
    s = launch_fwd(g, Q, K, V, cnt, idx, O, o_dtype == SA_F32, lse_or_null, false,
                   reinterpret_cast<cudaStream_t>(stream));
    if (s != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_quantize_fp8(const sa_shape* shape, const void* Q, const void* K, uint8_t* Q8, uint8_t* K8,
                                   float* q_scale, float* k_scale, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if (!Q || !K || !Q8 || !K8 || !q_scale || !k_scale)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, Q8, K8, q_scale, k_scale");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(Q8) || !aligned16(K8) || !aligned16(q_scale) ||
        !aligned16(k_scale))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    dim3 grid(g.n_q + g.n_k, g.BH);
    auto* q = reinterpret_cast<const __nv_bfloat16*>(Q);
    auto* k = reinterpret_cast<const __nv_bfloat16*>(K);
    if (g.d == 128)
        sa::fp8::quantize_kernel<128><<<grid, sa::fp8::QUANT_THREADS, 0, st>>>(q, k, Q8, K8, q_scale, k_scale, g.N,
                                                                               g.bq, g.bk, g.n_q, g.n_k);
    else
        sa::fp8::quantize_kernel<64><<<grid, sa::fp8::QUANT_THREADS, 0, st>>>(q, k, Q8, K8, q_scale, k_scale, g.N,
                                                                              g.bq, g.bk, g.n_q, g.n_k);
    if ((s = cuda_check(cudaGetLastError(), "quantize_kernel launch")) != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_fwd_fp8(const sa_shape* shape, const uint8_t* Q8, const uint8_t* K8, const float* q_scale,
                              const float* k_scale, const void* V, const int32_t* cnt, const int32_t* idx, void* O,
                              int o_dtype, float* lse_or_null, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_fwd_args(shape, Q8, K8, V, cnt, idx, O, o_dtype, lse_or_null, g)) != SA_OK) return s;
    if (g.d != 128) return fail(SA_ERR_UNSUPPORTED, "d=%d: the FP8 path supports d = 128", g.d);
    if (!q_scale || !k_scale) return fail(SA_ERR_INVALID_ARG, "NULL q_scale or k_scale");
    if (!aligned16(q_scale) || !aligned16(k_scale))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    Fp8Scales sc;
    sc.q = q_scale;
    sc.k = k_scale;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool f32 = o_dtype == SA_F32;
    s = (g.bq == 128)
            ? launch_attn_t<128, 128, true>(g, Q8, K8, V, cnt, idx, O, f32, lse_or_null, false, st, AttnTestKnobs(), sc)
            : launch_attn_t<128, 64, true>(g, Q8, K8, V, cnt, idx, O, f32, lse_or_null, false, st, AttnTestKnobs(), sc);
    if (s != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_test_fwd_withheld_copy(const sa_shape* shape, const void* Q, const void* K,
                                             const void* V, const int32_t* cnt, const int32_t* idx,
                                             void* O, int o_dtype, uint64_t wait_limit_ns,
                                             void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_fwd_args(shape, Q, K, V, cnt, idx, O, o_dtype, nullptr, g)) != SA_OK) return s;
    if (wait_limit_ns < 1000000ull || wait_limit_ns > WAIT_LIMIT_NS)
        return fail(SA_ERR_INVALID_ARG, "wait_limit_ns=%llu outside [1e6, 4e9]",
                    (unsigned long long)wait_limit_ns);
    AttnTestKnobs knobs;
    knobs.wait_limit_ns = wait_limit_ns;
    knobs.withhold_first_k = 1;
    s = launch_fwd(g, Q, K, V, cnt, idx, O, o_dtype == SA_F32, nullptr, false,
                   reinterpret_cast<cudaStream_t>(stream), knobs);
    if (s != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_fwd_dense(const sa_shape* shape, const void* Q, const void* K, const void* V,
                                void* O, int o_dtype, float* lse_or_null, void* stream) {
    Dims g;
    sa_status s;
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_out_dtype(o_dtype)) != SA_OK) return s;
    if (!Q || !K || !V || !O) return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, V, O");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
        (lse_or_null && !aligned16(lse_or_null)))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    // The dense path reads no index list.
    s = launch_fwd(g, Q, K, V, nullptr, nullptr, O, o_dtype == SA_F32, lse_or_null, true,
                   reinterpret_cast<cudaStream_t>(stream));
    if (s != SA_OK) return s;
    return ok();
}

sa_status sparse_attn_check_device_error(void* stream) {
    sa_status s = cuda_check(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)),
                             "stream synchronize");
    if (s != SA_OK) return s;
    sa::DeviceError rec;
    if ((s = cuda_check(cudaMemcpyFromSymbol(&rec, sa::g_device_error, sizeof(rec)),
                        "read device error record")) != SA_OK)
        return s;
    if (rec.code == 0) return ok();
    const sa::DeviceError zero = {0, 0, 0, 0};
    if ((s = cuda_check(cudaMemcpyToSymbol(sa::g_device_error, &zero, sizeof(zero)),
                        "clear device error record")) != SA_OK)
        return s;
    return fail((sa_status)rec.code, "device error %u (info 0x%x) in block %u, thread %u", rec.code,
                rec.info, rec.block, rec.thread);
}

// ------------------------------------------------- host-buffer pipeline
}  // extern "C"

namespace {

// Chunk geometry and device-buffer layout of sparse_attn_host.
struct HostPlan {
    Dims g;
    int hpc;             // heads per chunk
    int nchunk;
    size_t esize_o;      // bytes per O element
    size_t qkv_bytes;    // one chunk of Q (or K, or V)
    size_t o_bytes, cnt_bytes, idx_bytes, mws_bytes;
    size_t off_q[2], off_k[2], off_v[2], off_o[2], off_cnt[2], off_idx[2], off_mws[2];
    size_t total;
};

constexpr int HOST_MIN_ROWS_PER_CHUNK = 2368;   // ~8 query-block rows per attention pipeline on 148 SMs

// Heads of the next chunk when `rest` heads remain: full chunks of `hpc`
// heads while at least two chunks' worth remain, then halving chunks. The
// copies cross PCIe back to back while the compute of earlier chunks runs
// under them; what the pipeline cannot hide is the compute and copy-out of
// the last chunk, so the tail is made small.
int chunk_heads(int rest, int hpc) {
    if (rest >= 2 * hpc) return hpc;
    const int c = (rest + 1) / 2;
    return c < 1 ? 1 : (c > hpc ? hpc : c);
}

sa_status host_plan(const sa_shape* shape, int o_dtype, int heads_per_chunk, HostPlan& hp) {
    sa_status s;
    if ((s = check_shape(shape, hp.g)) != SA_OK) return s;
    if ((s = check_out_dtype(o_dtype)) != SA_OK) return s;
    if (heads_per_chunk < 0) return fail(SA_ERR_INVALID_ARG, "heads_per_chunk=%d", heads_per_chunk);
    const Dims& g = hp.g;
    int hpc = heads_per_chunk;
    if (hpc == 0) hpc = (HOST_MIN_ROWS_PER_CHUNK + g.n_q - 1) / g.n_q;
    if (hpc > g.BH) hpc = g.BH;
    hp.hpc = hpc;
    hp.nchunk = 0;
    for (int bh0 = 0; bh0 < g.BH; bh0 += chunk_heads(g.BH - bh0, hpc)) ++hp.nchunk;
    hp.esize_o = (o_dtype == SA_F32) ? 4 : 2;
    const size_t tok = (size_t)hpc * g.N * g.d;
    hp.qkv_bytes = tok * 2;
    hp.o_bytes = tok * hp.esize_o;
    hp.cnt_bytes = (size_t)hpc * g.n_q * 4;
    hp.idx_bytes = (size_t)hpc * g.n_q * g.n_k * 4;
    Dims sub = g;
    sub.B = 1;
    sub.H = hpc;
    sub.BH = hpc;
    hp.mws_bytes = workspace_layout(sub).total;
    size_t off = 0;
    for (int b = 0; b < 2; ++b) {
        hp.off_q[b] = off; off += round256(hp.qkv_bytes);
        hp.off_k[b] = off; off += round256(hp.qkv_bytes);
        hp.off_v[b] = off; off += round256(hp.qkv_bytes);
        hp.off_o[b] = off; off += round256(hp.o_bytes);
        hp.off_cnt[b] = off; off += round256(hp.cnt_bytes);
        hp.off_idx[b] = off; off += round256(hp.idx_bytes);
        hp.off_mws[b] = off; off += round256(hp.mws_bytes);
    }
    hp.total = off;
    return SA_OK;
}

// The library's three streams on the current device (copy-in, compute,
// copy-out), created on first use and kept for the life of the process.
sa_status host_streams(cudaStream_t (&out)[3]) {
    static std::mutex mu;
    static cudaStream_t streams[64][3] = {};
    int dev = 0;
    sa_status s;
    if ((s = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) != SA_OK) return s;
    if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 3; ++i) {
        if (!streams[dev][i] &&
            (s = cuda_check(cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking),
                            "create a pipeline stream")) != SA_OK)
            return s;
        out[i] = streams[dev][i];
    }
    return SA_OK;
}

// Events of one call, destroyed when the call returns (a destroyed event
// that is still pending completes normally).
struct CallEvents {
    cudaEvent_t ev[7] = {};
    ~CallEvents() {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
    }
    sa_status create() {
        for (cudaEvent_t& e : ev) {
            sa_status s = cuda_check(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "create an event");
            if (s != SA_OK) return s;
        }
        return SA_OK;
    }
};

}  // namespace

extern "C" {

size_t sparse_attn_host_workspace_bytes(const sa_shape* shape, int o_dtype, int heads_per_chunk) {
    HostPlan hp;
    if (host_plan(shape, o_dtype, heads_per_chunk, hp) != SA_OK) return 0;
    return hp.total;
}

sa_status sparse_attn_host(const sa_shape* shape, const void* Q, const void* K, const void* V, double k,
                           double p, void* O, int o_dtype, int32_t* cnt_or_null, int32_t* idx_or_null,
                           int heads_per_chunk, void* workspace, size_t workspace_bytes, void* stream) {
    HostPlan hp;
    sa_status s;
    if ((s = host_plan(shape, o_dtype, heads_per_chunk, hp)) != SA_OK) return s;
    if ((s = check_kp(k, p)) != SA_OK) return s;
    if (!Q || !K || !V || !O || !workspace)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, V, O, workspace");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
        (cnt_or_null && !aligned16(cnt_or_null)) || (idx_or_null && !aligned16(idx_or_null)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required; 256 for workspace)");
    if (workspace_bytes < hp.total)
        return fail(SA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, hp.total);
    cudaStream_t ps[3];
    if ((s = host_streams(ps)) != SA_OK) return s;
    const cudaStream_t s_in = ps[0], s_comp = ps[1], s_out = ps[2];
    const cudaStream_t caller = reinterpret_cast<cudaStream_t>(stream);
    CallEvents E;
    if ((s = E.create()) != SA_OK) return s;
    cudaEvent_t ev_start = E.ev[0], ev_in[2] = {E.ev[1], E.ev[2]}, ev_comp[2] = {E.ev[3], E.ev[4]},
                ev_out[2] = {E.ev[5], E.ev[6]};
    const Dims& g = hp.g;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    // Start after the caller's stream.
    if ((s = cuda_check(cudaEventRecord(ev_start, caller), "record the start event")) != SA_OK) return s;
    for (cudaStream_t st : ps)
        if ((s = cuda_check(cudaStreamWaitEvent(st, ev_start, 0), "order after the caller's stream")) != SA_OK)
            return s;
    const size_t tok_bytes = (size_t)g.N * g.d * 2;   // one head of Q, K or V
    int bh0 = 0;
    for (int c = 0; c < hp.nchunk; bh0 += chunk_heads(g.BH - bh0, hp.hpc), ++c) {
        const int b = c & 1;
        const int hc = chunk_heads(g.BH - bh0, hp.hpc);
        const sa_shape sub = {1, hc, g.N, g.d, g.bq, g.bk};
        void* Qd = ws + hp.off_q[b];
        void* Kd = ws + hp.off_k[b];
        void* Vd = ws + hp.off_v[b];
        void* Od = ws + hp.off_o[b];
        int32_t* cntd = reinterpret_cast<int32_t*>(ws + hp.off_cnt[b]);
        int32_t* idxd = reinterpret_cast<int32_t*>(ws + hp.off_idx[b]);
        const size_t in_bytes = (size_t)hc * tok_bytes;
        // Copy in, once the compute of chunk c-2 no longer reads buffer b.
        if (c >= 2 && (s = cuda_check(cudaStreamWaitEvent(s_in, ev_comp[b], 0), "order copy-in")) != SA_OK) return s;
        if ((s = cuda_check(cudaMemcpyAsync(Qd, static_cast<const uint8_t*>(Q) + (size_t)bh0 * tok_bytes, in_bytes,
                                            cudaMemcpyHostToDevice, s_in), "copy Q in")) != SA_OK ||
            (s = cuda_check(cudaMemcpyAsync(Kd, static_cast<const uint8_t*>(K) + (size_t)bh0 * tok_bytes, in_bytes,
                                            cudaMemcpyHostToDevice, s_in), "copy K in")) != SA_OK ||
            (s = cuda_check(cudaMemcpyAsync(Vd, static_cast<const uint8_t*>(V) + (size_t)bh0 * tok_bytes, in_bytes,
                                            cudaMemcpyHostToDevice, s_in), "copy V in")) != SA_OK ||
            (s = cuda_check(cudaEventRecord(ev_in[b], s_in), "record copy-in")) != SA_OK)
            return s;
        // Compute, once chunk c is in and the copy-out of chunk c-2 has read buffer b.
        if ((s = cuda_check(cudaStreamWaitEvent(s_comp, ev_in[b], 0), "order compute")) != SA_OK) return s;
        if (c >= 2 && (s = cuda_check(cudaStreamWaitEvent(s_comp, ev_out[b], 0), "order compute")) != SA_OK) return s;
        if ((s = sparse_attn_mask(&sub, Qd, Kd, k, p, cntd, idxd, nullptr, nullptr, ws + hp.off_mws[b], s_comp)) != SA_OK)
            return s;
        if ((s = sparse_attn_fwd(&sub, Qd, Kd, Vd, cntd, idxd, Od, o_dtype, nullptr, s_comp)) != SA_OK) return s;
        if ((s = cuda_check(cudaEventRecord(ev_comp[b], s_comp), "record compute")) != SA_OK) return s;
        // Copy out.
        if ((s = cuda_check(cudaStreamWaitEvent(s_out, ev_comp[b], 0), "order copy-out")) != SA_OK) return s;
        if ((s = cuda_check(cudaMemcpyAsync(static_cast<uint8_t*>(O) + (size_t)bh0 * g.N * g.d * hp.esize_o, Od,
                                            (size_t)hc * g.N * g.d * hp.esize_o, cudaMemcpyDeviceToHost, s_out),
                            "copy O out")) != SA_OK)
            return s;
        if (cnt_or_null &&
            (s = cuda_check(cudaMemcpyAsync(cnt_or_null + (size_t)bh0 * g.n_q, cntd, (size_t)hc * g.n_q * 4,
                                            cudaMemcpyDeviceToHost, s_out), "copy cnt out")) != SA_OK)
            return s;
        if (idx_or_null &&
            (s = cuda_check(cudaMemcpyAsync(idx_or_null + (size_t)bh0 * g.n_q * g.n_k, idxd,
                                            (size_t)hc * g.n_q * g.n_k * 4, cudaMemcpyDeviceToHost, s_out),
                            "copy idx out")) != SA_OK)
            return s;
        if ((s = cuda_check(cudaEventRecord(ev_out[b], s_out), "record copy-out")) != SA_OK) return s;
    }
    // The caller's stream waits for the last copy-out (the copy-out stream is
    // in order, and it waited for every compute, which waited for every copy-in).
    if ((s = cuda_check(cudaStreamWaitEvent(caller, ev_out[(hp.nchunk - 1) & 1], 0), "order the caller's stream")) != SA_OK)
        return s;
    return ok();
}

const char* sparse_attn_last_error(void) { return t_last_error.c_str(); }

const char* sparse_attn_version(void) { return "sparse_attn 0.1 (sm_100a)"; }

}  // extern "C"
