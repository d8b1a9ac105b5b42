/*
 * sparse_attn.h - C ABI of the hybrid Top-k+Top-p block-sparse attention
 * library (libsparse_attn.so), written for NVIDIA B200 (sm_100a).
 *
 * The method is the one summarised in "SpargeAttention2: Trainable Sparse
 * Attention via Hybrid Top-k+Top-p Masking and Distillation Fine-Tuning"
 * (gist.science summaries, Hindi and Arabic):
 *   §1 Problem Statement   - the Top-k rule (keep the top k of a row) and the
 *                            Top-p rule (keep entries until their cumulative
 *                            probability reaches p), and where each fails;
 *   §2A Hybrid Masking     - per row, keep the union of both selections;
 *   §2C Kernel             - a FlashAttention-style kernel applies that mask
 *                            per tile and skips the matmul and softmax of
 *                            masked tiles.
 * The block scores come from mean-pooled queries and keys, as in "SLA2:
 * Sparse-Linear Attention with Learnable Routing and QAT" §1 and §2B (a
 * compressed score from pooled Q and K) and "Sparse VideoGen2" §1 (mean
 * pooling of contiguous token blocks).
 *
 * Entry points (each documented at its declaration below)
 * ---------------------------------------------------------
 *   sparse_attn_mask[_noalloc]       steps 1-3: pooled scores, hybrid lists
 *   sparse_attn_select               step 3 alone, on given scores
 *   sparse_attn_fwd[_dense]          step 4 over the lists (or every block)
 *   sparse_attn_fused                steps 1-4 in one cooperative launch
 *   sparse_attn_quantize_fp8,
 *   sparse_attn_fwd_fp8              step 4 with e4m3 Q and K (per-block scales)
 *   sparse_attn_sparse_linear        SLA2's alpha mix with a linear branch
 *   sparse_attn_kmeans_permutation,
 *   sparse_attn_permute_rows         Sparse VideoGen2's semantic permutation
 *   sparse_attn_bwd                  gradients of step 4, lists held fixed
 *   sparse_attn_host                 steps 1-4 on host buffers, pipelined
 *   *_workspace_bytes, sparse_attn_check_device_error, sparse_attn_last_error,
 *   sparse_attn_version
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are dense, row-major, with no padding:
 *     Q, K, V      bf16  [B, H, N, d]     (token-major within a head)
 *     O            bf16 or fp32 [B, H, N, d]
 *     cnt          int32 [B, H, n_q]
 *     idx          int32 [B, H, n_q, n_k] (row capacity n_k)
 *     mask         uint8 [B, H, n_q, n_k]
 *     P            fp32  [B, H, n_q, n_k]
 *     lse          fp32  [B, H, N]        (natural log)
 *   where n_q = ceil(N / bq) and n_k = ceil(N / bk).
 * - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *   caller allocates and owns every buffer. The library allocates no memory
 *   per call; it keeps one small device error record per loaded module (and,
 *   once sparse_attn_host has run on a device, three streams there).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream). Calls only enqueue work; results are ready when the stream is.
 * - Supported shapes: d in {64, 128}; bq in {64, 128}; bk = 64;
 *   1 <= N, n_k <= 8192; B*H <= 65535. Pointers must be 16-byte aligned.
 * - Return value: SA_OK, or an error code with a message readable through
 *   sparse_attn_last_error() (thread-local). Argument errors are detected on
 *   the host before anything is enqueued. Errors raised inside a kernel
 *   (a bounded wait that ran out, an index out of range) are recorded on the
 *   device and reported by sparse_attn_check_device_error().
 * - Inputs must be finite; NaN or Inf propagation is unspecified.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, k/p out of range, misaligned */
    SA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set above */
    SA_ERR_CUDA = 3,          /* a CUDA runtime or driver call failed */
    SA_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out (device side) */
    SA_ERR_DEVICE_ASSERT = 5  /* a kernel found an invalid index list (device side) */
} sa_status;

typedef struct {
    int32_t B, H, N, d, bq, bk;
} sa_shape;

/* Element type of the attention output O. */
typedef enum {
    SA_BF16 = 0,  /* bf16, the fp32 result rounded to nearest even */
    SA_F32 = 1    /* fp32, the kernel's result before that rounding */
} sa_dtype;

/* Bytes of device workspace sparse_attn_mask needs for `shape` (pooled Q and
 * K, and the fp32 block-logit matrix). 0 on an invalid shape. */
size_t sparse_attn_mask_workspace_bytes(const sa_shape* shape);

/* Steps 1-3 of the path: block mask from Q and K.
 *   1. Qbar_i / Kbar_j = mean of the valid tokens of query block i (bq
 *      tokens) and key block j (bk tokens);
 *   2. P = row softmax of Qbar Kbar^T / sqrt(d), fp32;
 *   3. per row, keep the union of the Top-k set (the ceil(k * n_k) highest
 *      scores; k >= 1 keeps all) and the Top-p set (the shortest prefix of
 *      the score order whose mass reaches p of the row total; p >= 1 keeps
 *      all). The score order is by P descending, equal scores by lower
 *      index; mass is counted in 31-bit fixed point, floor(P * 2^31), and
 *      the target is ceil(p * W) in double, W the row's fixed-point total.
 *      The selection is exact given P: any order of the reductions gives the
 *      same kept set.
 * Inputs:  Q, K bf16 [B,H,N,d]; k, p in [0, 1], not both 0.
 * Outputs: cnt[b,h,i] = number of kept key blocks; idx[b,h,i,0:cnt] = kept
 *          key-block indices, ascending (entries past cnt are not written);
 *          mask (optional, may be NULL) = 1 for kept blocks, 0 otherwise;
 *          P_out (optional, may be NULL) = the fp32 scores the selection
 *          used.
 * workspace: device buffer of sparse_attn_mask_workspace_bytes(shape) bytes,
 *          256-byte aligned; its contents are scratch. */
sa_status sparse_attn_mask(const sa_shape* shape, const void* Q, const void* K,
                           double k, double p,
                           int32_t* cnt, int32_t* idx,
                           uint8_t* mask_or_null, float* P_out_or_null,
                           void* workspace, void* stream);

/* sparse_attn_mask without a caller-provided workspace, for callers that
 * cannot allocate device memory on their call path: for example a runtime
 * that has handed all device memory to its own pool, or a plugin or callback
 * context where a cudaMalloc is not allowed or would stall the device. It has
 * no counterpart in the papers; it is a packaging of the same computation.
 * Same arguments, outputs and selection as sparse_attn_mask, minus the
 * workspace. The scratch lives in one fixed device array inside the library,
 * SPARSE_ATTN_NOALLOC_SCRATCH_BYTES (32 MiB) per device, held by every GPU
 * that loads the library until the process exits. Shapes whose workspace
 * (sparse_attn_mask_workspace_bytes) exceeds it are rejected with
 * SA_ERR_UNSUPPORTED before anything is enqueued. The function allocates
 * nothing. The first call on a device looks up the array's device address
 * (a runtime call), so make that first call before any stream capture. All
 * calls share the array: calls whose work overlaps on the GPU (different
 * streams, or different host threads, without ordering between them) race
 * on it and give undefined results. Nothing in the array needs clearing:
 * each call writes every scratch byte it later reads. */
#define SPARSE_ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
sa_status sparse_attn_mask_noalloc(const sa_shape* shape, const void* Q, const void* K,
                                   double k, double p,
                                   int32_t* cnt, int32_t* idx,
                                   uint8_t* mask_or_null, float* P_out_or_null,
                                   void* stream);

/* Step 3 alone, on a caller-supplied fp32 score matrix P [B,H,n_q,n_k]
 * (rows of non-negative finite values). Same selection code and outputs as
 * sparse_attn_mask; used to check the selection bit for bit. */
sa_status sparse_attn_select(const sa_shape* shape, const float* P, double k, double p,
                             int32_t* cnt, int32_t* idx, uint8_t* mask_or_null,
                             void* stream);

/* Step 4: block-sparse attention over the kept tiles only (SpargeAttention2
 * §2C). For every query block i of every (b, h):
 *   O[rows of i] = softmax(Q_i K_u^T / sqrt(d)) V_u over the tokens u of the
 *   key blocks idx[b,h,i,0:cnt[b,h,i]] (tokens >= N excluded);
 * no work is issued for key blocks not in the list. A row with cnt = 0 gets
 * O = 0 and lse = -inf. Index entries must lie in [0, n_k); an entry outside
 * is skipped and reported as SA_ERR_DEVICE_ASSERT.
 * Inputs: Q, K, V bf16 [B,H,N,d]; cnt, idx as produced by sparse_attn_mask.
 * Outputs: O [B,H,N,d] of type o_dtype (SA_BF16 or SA_F32; the bf16 output
 *          is exactly the round-to-nearest-even of the fp32 one);
 *          lse (optional) fp32 [B,H,N], natural log of the softmax
 *          denominator of each query row. */
sa_status sparse_attn_fwd(const sa_shape* shape, const void* Q, const void* K, const void* V,
                          const int32_t* cnt, const int32_t* idx,
                          void* O, int o_dtype, float* lse_or_null, void* stream);

/* Step 4 with every key block kept (full attention through the same kernel;
 * no index list is read). The reference point for the sparse speed-up. */
sa_status sparse_attn_fwd_dense(const sa_shape* shape, const void* Q, const void* K,
                                const void* V, void* O, int o_dtype, float* lse_or_null,
                                void* stream);

/* Low-bit forward, step 1 of 2: per-block FP8 (e4m3) quantisation of Q and K.
 * "SLA2: Sparse-Linear Attention with Learnable Routing and QAT" §2C runs
 * the sparse branch in low-bit (INT8/FP8) attention; the page names neither
 * format nor scaling. Here: one fp32 scale per query block of Q (bq tokens)
 * and per key block of K (bk tokens), s = amax / 448 with amax the block's
 * largest |x| (fp32); each code is e4m3(x * (448 / amax)), products and
 * quotient in fp32 round-to-nearest, the conversion rounding to nearest even
 * and saturating at 448. An all-zero block gets s = 0 and zero codes.
 * Inputs:  Q, K bf16 [B,H,N,d].
 * Outputs: Q8, K8 e4m3 codes [B,H,N,d] (one byte each); q_scale fp32
 *          [B,H,n_q]; k_scale fp32 [B,H,n_k]. */
sa_status sparse_attn_quantize_fp8(const sa_shape* shape, const void* Q, const void* K,
                                   uint8_t* Q8, uint8_t* K8, float* q_scale, float* k_scale,
                                   void* stream);

/* Low-bit forward, step 2 of 2: sparse_attn_fwd with the score product in
 * FP8. S = Q K^T runs on the tensor cores in e4m3 (tcgen05 kind::f8f6f4) and
 * is rescaled per tile by q_scale[i] * k_scale[j]; P and V stay in the bf16
 * path of sparse_attn_fwd (on B200 the exponentials of P already take as long
 * per tile as the bf16 P V product, so an FP8 P V would not shorten a tile).
 * Same kept-tile semantics, outputs and error reporting as sparse_attn_fwd.
 * Inputs: Q8, K8, q_scale, k_scale from sparse_attn_quantize_fp8; V bf16
 *         [B,H,N,d]; cnt, idx as for sparse_attn_fwd. d must be 128
 *         (SA_ERR_UNSUPPORTED otherwise).
 * Outputs: O [B,H,N,d] of type o_dtype; lse (optional) fp32 [B,H,N]. */
sa_status sparse_attn_fwd_fp8(const sa_shape* shape, const uint8_t* Q8, const uint8_t* K8,
                              const float* q_scale, const float* k_scale, const void* V,
                              const int32_t* cnt, const int32_t* idx,
                              void* O, int o_dtype, float* lse_or_null, void* stream);

/* Bytes of device workspace sparse_attn_fused needs for `shape`: the fp32
 * block means of Q and K (4 * B*H*(n_q + n_k)*d, each part rounded up to
 * 256) and a 256-byte grid-barrier counter. 0 on an invalid shape or one
 * the single launch does not support (see below). */
size_t sparse_attn_fused_workspace_bytes(const sa_shape* shape);

/* Steps 1-4 in ONE kernel launch: "SpargeAttention2" §2C (Efficient Kernel
 * Implementation) applies the block mask inside the FlashAttention-style
 * kernel. The launch is cooperative (every CTA resident at once) and runs
 * three phases separated by grid barriers: the block means of Q and K (as
 * sparse_attn_mask step 1), then the scores and hybrid Top-k + Top-p lists
 * of every query-block row (steps 2-3, a tile of 12 rows at a time in
 * shared memory), then the block-sparse attention over those lists (step
 * 4, as sparse_attn_fwd). Every phase takes the same operations in the same
 * order as the separate entry points, so cnt, idx, O and lse are bit-equal
 * to sparse_attn_mask followed by sparse_attn_fwd.
 * Inputs:  Q, K, V bf16 [B,H,N,d]; k, p as for sparse_attn_mask.
 * Outputs: cnt int32 [B,H,n_q] and idx int32 [B,H,n_q,n_k] (entries past
 *          cnt unspecified), O [B,H,N,d] of type o_dtype, lse fp32 [B,H,N]
 *          or NULL.
 * workspace: device, sparse_attn_fused_workspace_bytes(shape) bytes,
 *          256-byte aligned; workspace_bytes is checked against that size.
 *          The grid counter in it is zeroed by a memset on `stream` before
 *          the kernel, so calls that overlap on the GPU need separate
 *          workspaces.
 * Limits:  the selection phase holds 12 rows of n_k logits and fixed-point
 *          masses in the attention kernel's shared memory: n_k <= 1549 for
 *          d = 128 (N <= 99,136 tokens) and n_k <= 1344 for d = 64
 *          (N <= 86,016); larger shapes get SA_ERR_UNSUPPORTED.
 * Errors:  as sparse_attn_mask and sparse_attn_fwd; a grid barrier that
 *          waits past the kernels' bound (4 s) is reported as SA_ERR_TIMEOUT
 *          by sparse_attn_check_device_error and the attention phase is
 *          skipped. */
sa_status sparse_attn_fused(const sa_shape* shape, const void* Q, const void* K, const void* V,
                            double k, double p, int32_t* cnt, int32_t* idx, void* O, int o_dtype,
                            float* lse_or_null, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Bytes of device workspace sparse_attn_kmeans_permutation needs: the
 * cluster offsets, 4 * B*H*(C + 1) rounded up to 256. 0 on an invalid shape
 * or C. */
size_t sparse_attn_kmeans_workspace_bytes(const sa_shape* shape, int C);

/* Semantic-aware permutation of "Sparse VideoGen2: Accelerate Video
 * Generation with Sparse Attention via Semantic-Aware Permutation" §2A: the
 * N token vectors of every (b, h) are clustered by k-means into C clusters
 * and listed cluster by cluster, so that a block of the permuted sequence
 * holds tokens of one cluster (Q and K are permuted independently; V takes
 * K's permutation). §2C starts k-means from the previous step's centroids:
 * init_or_null. The page fixes no initialisation, distance or tie rule; here
 * (so that the result is exact and reproducible):
 *   start     centroid c = the token at floor(c N / C), unless init is given;
 *   assign    squared Euclidean distance summed over the channels in order,
 *             each subtraction, product and addition rounded to fp32 (no
 *             fused multiply-add); the nearest centroid, ties to the lower
 *             index;
 *   update    the fp32 sum of a cluster's members in ascending token order,
 *             divided by their count; an empty cluster keeps its centroid;
 *   iters     `iters` rounds of (assign, update), then a final assign;
 *   perm      tokens sorted by final cluster id, ascending token order within
 *             a cluster (a stable sort): perm[i] is the token at position i.
 * Inputs:  shape (B, H, N, d with d in {64, 128}; bq and bk are checked as
 *          elsewhere but unused); X bf16 [B,H,N,d]; C clusters, 1 <= C <=
 *          min(N, 8192); iters in [0, 100]; init_or_null fp32 [B,H,C,d].
 * Outputs: ids int32 [B,H,N] (final cluster of every token), perm int32
 *          [B,H,N], centroids fp32 [B,H,C,d] (after `iters` updates; may be
 *          the same buffer as init_or_null, which is then updated in place;
 *          any other overlap of the two is not allowed).
 * workspace: device, sparse_attn_kmeans_workspace_bytes(shape, C) bytes,
 *          256-byte aligned; workspace_bytes is checked against that size.
 * Device pointers 16-byte aligned. Errors: SA_ERR_INVALID_ARG on a bad
 * shape, C, iters, pointer or workspace; SA_ERR_CUDA on a failed launch. */
sa_status sparse_attn_kmeans_permutation(const sa_shape* shape, const void* X, int C, int iters,
                                         const float* init_or_null, int32_t* ids, int32_t* perm,
                                         float* centroids, void* workspace, size_t workspace_bytes,
                                         void* stream);

/* Row permutation of [B,H,N,d] for the semantic-aware permutation (Sparse
 * VideoGen2 §2A): inverse = 0 gathers Y[b,h,i] = X[b,h,perm[b,h,i]] (tokens
 * into cluster order), inverse = 1 scatters Y[b,h,perm[b,h,i]] = X[b,h,i]
 * (an output in cluster order back to token order). Rows are copied bit for
 * bit. dtype: SA_BF16 or SA_F32, the element type of X and Y. perm must be a
 * permutation of 0..N-1 for every (b, h) (the result of
 * sparse_attn_kmeans_permutation); an entry outside [0, N) is skipped and
 * reported as SA_ERR_DEVICE_ASSERT by sparse_attn_check_device_error (a
 * repeated entry leaves some rows of Y unwritten and is not detected).
 * X and Y distinct, device pointers 16-byte aligned.
 * Errors: SA_ERR_INVALID_ARG on a bad shape, dtype or pointer. */
sa_status sparse_attn_permute_rows(const sa_shape* shape, const void* X, const int32_t* perm,
                                   void* Y, int dtype, int inverse, void* stream);

/* Bytes of device workspace sparse_attn_sparse_linear needs for `shape`:
 * phi(Q) and phi(K) in bf16 (2 * 2 * B*H*N*d), per-key-block sums of phi(k)
 * (4 * B*H*ceil(N/64)*d), split partial states (4 * B*H*splits*d*d, splits
 * about 148 / (B*H), at least 1), the state as a bf16 pair (2 * 2 * B*H*d*d)
 * and z (4 * B*H*d), each rounded up to 256 bytes. 0 on an invalid shape or
 * d != 128. */
size_t sparse_attn_sparse_linear_workspace_bytes(const sa_shape* shape);

/* The sparse + linear combination of "SLA2: Sparse-Linear Attention with
 * Learnable Routing and QAT" §2A: O = alpha * O_s + (1 - alpha) * O_l, where
 * O_s is the sparse branch (sparse_attn_fwd over the kept blocks, passed in)
 * and O_l is linear attention over the complement of a row's kept blocks.
 * The page prints no feature map; here phi(x) = elu(x) + 1 (positive), and
 * for a query token t of query block i,
 *   O_l(t) = sum_u (phi(q_t) . phi(k_u)) v_u / sum_u phi(q_t) . phi(k_u)
 * over the valid key tokens u of the key blocks NOT in idx[i, 0:cnt[i]];
 * O_l = 0 for a row that keeps every key block. It is computed as the total
 * over all keys minus the kept part: the per-head state H = phi(K)^T V and
 * z = sum_u phi(k_u) are built on the tensor cores (phi rounded to bf16, the
 * operands of every product), and each row subtracts its kept tiles' sums
 * inside the same fp32 accumulator. The result loses relative precision
 * when the complement carries only a small part of the row's total linear
 * weight (the subtraction cancels); on the workloads here it keeps at least
 * 5% of it.
 * Inputs:  Q, K, V bf16 [B,H,N,d] (d = 128, else SA_ERR_UNSUPPORTED); cnt,
 *          idx as for sparse_attn_fwd; O_s [B,H,N,d] of type o_dtype (the
 *          sparse branch's output); alpha fp32 [B,H,N], values in [0, 1].
 * Output:  O [B,H,N,d] of type o_dtype.
 * workspace: device, sparse_attn_sparse_linear_workspace_bytes(shape) bytes,
 *          256-byte aligned; workspace_bytes is checked against that size. */
sa_status sparse_attn_sparse_linear(const sa_shape* shape, const void* Q, const void* K,
                                    const void* V, const int32_t* cnt, const int32_t* idx,
                                    const void* O_s, const float* alpha, void* O, int o_dtype,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace sparse_attn_bwd needs for `shape`: the per-row
 * log-sum-exp and D = rowsum(dO * O) (8 * B*H * n_q * bq bytes), the
 * kept-block bitmap (4 * B*H * n_q * ceil(n_k/32)), and the transposed lists
 * (4 * B*H * ceil(n_k/2) * (n_q + 1)), each rounded up to 256 bytes.
 * 0 on an invalid shape. */
size_t sparse_attn_bwd_workspace_bytes(const sa_shape* shape);

/* Backward pass of step 4: the gradients of sparse_attn_fwd's output with the
 * kept-block lists held fixed. SpargeAttention2 §2B (Velocity Distillation
 * Fine-Tuning) fine-tunes the model through the sparse attention of §2C;
 * the pages give no formula, so this is the plain derivative of the forward
 * (the selection of §2A is piecewise constant in Q and K and carries none).
 * For every query block i with kept key tokens u, c = 1/sqrt(d) and
 * P = softmax(c Q_i K_u^T) (recomputed from lse):
 *   dV_u += P^T dO_i;  dS = P * (dO_i V_u^T - D_i), D_i = rowsum(dO_i * O_i);
 *   dQ_i = c dS K_u;   dK_u += c dS^T Q_i.
 * A key token that no query block keeps gets dK = dV = 0; a query block with
 * cnt = 0 gets dQ = 0.
 * Inputs:  Q, K, V bf16 [B,H,N,d] (those of the forward); O bf16 [B,H,N,d]
 *          and lse fp32 [B,H,N], the forward's bf16 output and log-sum-exp;
 *          dO bf16 [B,H,N,d], the gradient of the loss with respect to O;
 *          cnt, idx as given to the forward. A list must not repeat a block:
 *          a repeated or out-of-range entry is reported as
 *          SA_ERR_DEVICE_ASSERT and counted once (repeated) or skipped.
 * Outputs: dQ, dK, dV [B,H,N,d] of type g_dtype (SA_BF16 or SA_F32).
 * workspace: device buffer of sparse_attn_bwd_workspace_bytes(shape) bytes,
 *          256-byte aligned; its contents are scratch.
 * The sums are deterministic (no atomics): dQ is accumulated per query block
 * in list order, dK and dV per pair of adjacent key blocks in ascending
 * query-block order. */
sa_status sparse_attn_bwd(const sa_shape* shape, const void* Q, const void* K, const void* V,
                          const void* O, const void* dO, const float* lse,
                          const int32_t* cnt, const int32_t* idx,
                          void* dQ, void* dK, void* dV, int g_dtype,
                          void* workspace, void* stream);

/* Bytes of device workspace sparse_attn_host needs for `shape` with chunks of
 * `heads_per_chunk` (b, h) heads (0 = the library's choice, see below): two
 * device copies of a chunk of Q, K, V and O (O in the element type o_dtype),
 * of its cnt and idx, and of the mask workspace of a chunk. 0 on an invalid
 * shape, o_dtype or heads_per_chunk. */
size_t sparse_attn_host_workspace_bytes(const sa_shape* shape, int o_dtype, int heads_per_chunk);

/* The whole path (steps 1-4: sparse_attn_mask, then sparse_attn_fwd) on HOST
 * buffers. It has no counterpart in the papers: it packages the same
 * computation for callers whose Q, K, V are in host memory, overlapping the
 * PCIe copies with the GPU work. The (b, h) heads are independent rows of the
 * mask and of the attention, so they are processed in chunks of at most
 * heads_per_chunk heads (0 = enough heads for at least 2,368 query-block rows
 * per chunk, about 8 rows per attention pipeline of a B200); once fewer than
 * two full chunks remain, each chunk takes half of the remaining heads
 * (rounded up), so that the last chunk, whose compute and copy-out nothing
 * overlaps, is small. While chunk c is computed, chunk c+1 is copied to the
 * device and chunk c-1's results back to the host, on three streams owned by
 * the library, with two device copies of every chunk buffer (in
 * `workspace`). The results are those of the device entry points on the whole
 * tensors, bit for bit.
 * Host pointers: Q, K, V bf16 [B,H,N,d]; O [B,H,N,d] of type o_dtype; cnt
 *          int32 [B,H,n_q] and idx int32 [B,H,n_q,n_k] (each may be NULL: not
 *          copied back). They must be page-locked (cudaHostAlloc or
 *          cudaHostRegister) for the copies to run asynchronously; pageable
 *          memory works but each copy then blocks the host. 16-byte aligned.
 * workspace: device, sparse_attn_host_workspace_bytes(shape, o_dtype,
 *          heads_per_chunk) bytes, 256-byte aligned; workspace_bytes is
 *          checked against that size.
 * Ordering: the call's work starts after the work already in `stream` and
 *          `stream` waits for all of it; host buffers may be read or written
 *          by the host only once `stream` has reached that point. An error
 *          returned after the first chunk was enqueued leaves earlier chunks'
 *          copies in flight (they finish on their own). */
sa_status sparse_attn_host(const sa_shape* shape, const void* Q, const void* K, const void* V,
                           double k, double p, void* O, int o_dtype,
                           int32_t* cnt_or_null, int32_t* idx_or_null, int heads_per_chunk,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, returns the first device-side error recorded since
 * the last call (SA_OK if none) and clears the record. */
sa_status sparse_attn_check_device_error(void* stream);

/* Message of the last error returned on this host thread ("" if none). */
const char* sparse_attn_last_error(void);

/* Library version string. */
const char* sparse_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
