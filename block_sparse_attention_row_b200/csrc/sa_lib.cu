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
// `rows` tokens x 1 head, 128-byte swizzle; out-of-range rows read as zero.
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

template <int D, int BQ>
sa_status launch_attn_t(const Dims& g, const void* Q, const void* K, const void* V, const int32_t* cnt,
                        const int32_t* idx, void* O, bool out_f32, float* lse, bool dense,
                        cudaStream_t st) {
    using L = sa::attn::Layout<D>;
    CUtensorMap mq, mk, mv;
    sa_status s;
    if ((s = make_map(&mq, Q, g, sa::attn::MROWS)) != SA_OK) return s;
    if ((s = make_map(&mk, K, g, sa::attn::BK)) != SA_OK) return s;
    if ((s = make_map(&mv, V, g, sa::attn::BK)) != SA_OK) return s;
    auto kern = sa::attn::sparse_attn_fwd_kernel<D, BQ>;
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
    prm.wait_limit_ns = WAIT_LIMIT_NS;
    // Persistent: one CTA per multiprocessor (fewer when there are fewer row pairs).
    const int pairs = (prm.rows + sa::attn::NSLOT - 1) / sa::attn::NSLOT;
    const int grid = pairs < sm_count() ? pairs : sm_count();
    kern<<<grid, sa::attn::NUM_THREADS, L::DYN_BYTES, st>>>(mq, mk, mv, prm);
    return cuda_check(cudaGetLastError(), "sparse_attn_fwd_kernel launch");
}

sa_status launch_fwd(const Dims& g, const void* Q, const void* K, const void* V, const int32_t* cnt,
                     const int32_t* idx, void* O, bool out_f32, float* lse, bool dense,
                     cudaStream_t st) {
    if (g.d == 128 && g.bq == 128)
        return launch_attn_t<128, 128>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st);
    if (g.d == 128 && g.bq == 64)
        return launch_attn_t<128, 64>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st);
    if (g.d == 64 && g.bq == 128)
        return launch_attn_t<64, 128>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st);
    return launch_attn_t<64, 64>(g, Q, K, V, cnt, idx, O, out_f32, lse, dense, st);
}

sa_status check_out_dtype(int o_dtype) {
    if (o_dtype != SA_BF16 && o_dtype != SA_F32)
        return fail(SA_ERR_INVALID_ARG, "o_dtype=%d (SA_BF16=0 or SA_F32=1)", o_dtype);
    return SA_OK;
}

__global__ void exp2_poly_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = sa::attn::exp2_poly(x[i]);
}

}  // namespace

extern "C" {

sa_status sparse_attn_test_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
    if (!x || !y || n < 0) return fail(SA_ERR_INVALID_ARG, "exp2 probe: bad arguments");
    if (n == 0) return ok();
    const int64_t blocks = (n + 255) / 256;
    if (blocks > 0x7FFFFFFF) return fail(SA_ERR_INVALID_ARG, "exp2 probe: n too large");
    exp2_poly_probe_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    sa_status s = cuda_check(cudaGetLastError(), "exp2 probe launch");
    return s != SA_OK ? s : ok();
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
    if ((s = check_shape(shape, g)) != SA_OK) return s;
    if ((s = check_out_dtype(o_dtype)) != SA_OK) return s;
    if (!Q || !K || !V || !cnt || !idx || !O)
        return fail(SA_ERR_INVALID_ARG, "NULL pointer among Q, K, V, cnt, idx, O");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(cnt) || !aligned16(idx) ||
        !aligned16(O) || (lse_or_null && !aligned16(lse_or_null)))
        return fail(SA_ERR_INVALID_ARG, "misaligned pointer (16 bytes required)");
    s = launch_fwd(g, Q, K, V, cnt, idx, O, o_dtype == SA_F32, lse_or_null, false,
                   reinterpret_cast<cudaStream_t>(stream));
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

const char* sparse_attn_last_error(void) { return t_last_error.c_str(); }

const char* sparse_attn_version(void) { return "sparse_attn 0.1 (sm_100a)"; }

}  // extern "C"
