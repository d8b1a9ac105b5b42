// sa_fp8_kernels.cuh - per-block FP8 (e4m3) quantisation of Q and K for the
// low-bit forward path.
//
// Method: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
// (gist.science summary) §2C: the sparse branch runs low-bit (INT8/FP8)
// attention. Reading taken (the page names neither format nor scaling): e4m3
// codes with one fp32 scale per block of tokens, s = amax / 448, code =
// e4m3(x * (448 / amax)) rounded to nearest even and saturated; an all-zero
// block gets s = 0 and zero codes. Q is scaled per query block, K per key
// block, so that a score tile S = Q_i K_j^T is recovered as s_i s_j (codes
// product).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sa_ptx.cuh"

namespace sa {
namespace fp8 {

constexpr int QUANT_THREADS = 128;

// Two fp32 values to two e4m3 codes (lo in the low byte), round to nearest
// even, saturated to the largest finite value.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One CTA per block: blockIdx.x in [0, n_q) a Q block of bq tokens, in
// [n_q, n_q + n_k) a K block of bk tokens; blockIdx.y = b*H + h. The block
// (at most 128 tokens x D channels of bf16) is read once into registers, its
// amax reduced, then its codes written.
template <int D>
__global__ void __launch_bounds__(QUANT_THREADS)
quantize_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, uint8_t* __restrict__ Q8,
                uint8_t* __restrict__ K8, float* __restrict__ q_scale, float* __restrict__ k_scale, int N, int bq,
                int bk, int n_q, int n_k) {
    constexpr int CG = D / 8;                    // 16-byte chunks per token row
    constexpr int RG = QUANT_THREADS / CG;       // token rows read in parallel
    constexpr int MAX_IT = 128 / RG;             // rows per thread for a 128-token block
    __shared__ float red[QUANT_THREADS / 32];
    const int bh = blockIdx.y;
    int blk = blockIdx.x;
    const __nv_bfloat16* X = Q;
    uint8_t* X8 = Q8;
    float* scale_out = q_scale + (size_t)bh * n_q + blk;
    int bs = bq;
    if (blk >= n_q) {
        blk -= n_q;
        X = K;
        X8 = K8;
        scale_out = k_scale + (size_t)bh * n_k + blk;
        bs = bk;
    }
    const int lo = blk * bs;
    const int valid = min(N - lo, bs);
    const size_t base = ((size_t)bh * N + lo) * D;
    const uint4* src = reinterpret_cast<const uint4*>(X + base);
    const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
    uint4 v[MAX_IT];
    float amax = 0.f;
#pragma unroll
    for (int it = 0; it < MAX_IT; ++it) {
        const int r = rg + it * RG;
        v[it] = r < valid ? __ldg(src + (size_t)r * CG + cg) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < QUANT_THREADS / 32; ++w) amax = fmaxf(amax, red[w]);
    const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
    if (threadIdx.x == 0) *scale_out = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
    uint2* dst = reinterpret_cast<uint2*>(X8 + base);
#pragma unroll
    for (int it = 0; it < MAX_IT; ++it) {
        const int r = rg + it * RG;
        if (r >= valid) break;
        const uint32_t w[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
        uint32_t packed[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float a0 = __fmul_rn(__uint_as_float(w[2 * e] << 16), inv);
            const float a1 = __fmul_rn(__uint_as_float(w[2 * e] & 0xFFFF0000u), inv);
            const float a2 = __fmul_rn(__uint_as_float(w[2 * e + 1] << 16), inv);
            const float a3 = __fmul_rn(__uint_as_float(w[2 * e + 1] & 0xFFFF0000u), inv);
            packed[e] = (uint32_t)cvt_e4m3x2(a0, a1) | ((uint32_t)cvt_e4m3x2(a2, a3) << 16);
        }
        dst[(size_t)r * CG + cg] = make_uint2(packed[0], packed[1]);
    }
}

}  // namespace fp8
}  // namespace sa
