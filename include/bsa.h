/*
 * bsa.h — C ABI of libbsa.so: training-free block-sparse attention for video DiTs
 * on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages; cited by title and section):
 *  [SBC]  "Sparse-block compensation" — mlx-arsenal research notes:
 *         §The problem, §SVG-EAR — centroid compensation, §SparsePR — probe-fitted
 *         residual repair, §What mlx-arsenal ships, §No LSE needed, §Recipe,
 *         §Deviations from the papers.
 *  [HMR]  "Dynamic block masks and head-wise mask reuse" — mlx-arsenal research
 *         notes: §XAttention — anti-diagonal block scoring, §HEART — head-wise
 *         temporal mask reuse, §What mlx-arsenal ships, §Recipe, §Deviations,
 *         §Out of scope (padding).
 *  [SPR]  "Partition the Support, Reconstruct the Residual: Training-Free Sparse
 *         Attention for Video Generation and World Models" — paper summary:
 *         probe-fitted residual reconstruction, group-major permutation, GQA.
 *
 * Conventions shared by every entry point
 *  - Tensors are caller-owned DEVICE memory, contiguous, row-major. Q is
 *    (B, Hq, S, D); K and V are (B, Hkv, S, D) with Hq a multiple of Hkv (query head
 *    h uses KV head h / (Hq / Hkv)). Element type: BSA_BF16 or BSA_F32.
 *  - Cluster labels are int32 device arrays shared by every batch and head.
 *    Masks are uint8 device arrays, 1 = block kept (computed exactly).
 *  - The library never allocates device memory. An op that needs scratch space
 *    has a *_workspace_bytes query; the caller passes a device buffer at least that
 *    large (256-byte aligned). Workspace contents are undefined on return.
 *  - Every call is asynchronous on the caller's stream (a cudaStream_t passed as
 *    void*, NULL = legacy default stream) unless its comment says it synchronises.
 *  - Return value: BSA_OK or a negative status. Argument errors are detected on the
 *    host before any launch. A device-side wait that runs out of time records
 *    BSA_ERR_TIMEOUT, read back with bsa_get_device_status().
 *  - Output attention tensors are fp32 (B, Hq, S, D) in the ORIGINAL token order.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = -1,   /* null pointer, bad size, inconsistent shapes */
  BSA_ERR_UNSUPPORTED = -2,   /* dtype, head dim or size outside the supported set */
  BSA_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed */
  BSA_ERR_TIMEOUT = -4,       /* a bounded device-side wait gave up */
  BSA_ERR_WORKSPACE = -5      /* workspace missing or too small */
};

enum { BSA_BF16 = 0, BSA_F32 = 1 };

/* Flags of bsa_centroid_compensated_attention_ex. */
enum { BSA_REUSE_PLAN = 1 };

/* Problem shape. Sq = Sk = S for self-attention; D in {64, 128}. */
typedef struct {
  int B, Hq, Hkv, Sq, Sk, D;
  int dtype; /* BSA_BF16 or BSA_F32 */
} bsa_shape;

/* Human-readable name of a status code (static string). */
const char* bsa_status_string(int status);

/* Copies the calling thread's last error detail (NUL-terminated) into buf. */
void bsa_last_error_detail(char* buf, size_t len);

/* Library version as major*10000 + minor*100 + patch. */
int bsa_version(void);

/*
 * Synchronises `stream`, then returns and clears the device status word: BSA_OK, or
 * BSA_ERR_TIMEOUT if a kernel's bounded wait gave up since the last call. *where
 * (nullable) receives the kernel-specific site code of the first failure.
 */
int bsa_get_device_status(void* stream, int* where);

/*
 * Check of the failure path every kernel's waits share (no counterpart on the pages):
 * launches one warp that waits, with the same bounded mbarrier wait the kernels use, on
 * a barrier that nothing ever arrives on. After `limit_ns` nanoseconds of wall time
 * (clamped to [1 us, 2 s]) the wait gives up, records BSA_ERR_TIMEOUT with site code
 * 90 in the device status word and the kernel returns normally, leaving the context
 * usable. Asynchronous on `stream`; read the outcome with bsa_get_device_status().
 * Returns BSA_ERR_CUDA if the launch fails. Allocates nothing.
 */
int bsa_wait_timeout_selftest(long long limit_ns, void* stream);

/* Number of kernel launches the library has made since it was loaded. */
long long bsa_launch_count(void);

/*
 * Kernel timing hooks. bsa_profile_enable(n) (n > 0) makes the next n launches of each
 * timed kernel record a CUDA event pair around the launch on its stream; n == 0 turns
 * timing off. bsa_profile_read(kernel, &ms, &count) synchronises those events and
 * returns the summed duration and the number of timed launches. kernel: 0 = the
 * attention kernel of centroid_compensated_attention, 1 = the scoring kernel,
 * 2 = the attention kernel of probe_dense_attention. Creates CUDA events (host
 * objects), no device memory.
 */
int bsa_profile_enable(int max_launches);
int bsa_profile_read(int kernel, float* total_ms, int* launches);

/*
 * tile_labels — [SBC] §What mlx-arsenal ships (tile_labels: labels matching Sliding
 * Tile Attention tiles), §Recipe. Token s = (t*H + h)*W + w of a T x H x W latent
 * grid gets label ((t/tt)*nH + h/th)*nW + w/tw with nH = ceil(H/th),
 * nW = ceil(W/tw); tiles at the far edges are partial when a tile size does not
 * divide its axis.
 *   labels     : device int32 (T*H*W), written.
 *   n_clusters : host int, written with ceil(T/tt)*nH*nW (nullable).
 * Errors: INVALID_ARG for non-positive sizes or a null labels pointer.
 */
int bsa_tile_labels(int T, int H, int W, int tt, int th, int tw, int32_t* labels,
                    int* n_clusters, void* stream);

/*
 * sliding_tile_block_mask — [SBC] §What mlx-arsenal ships (sliding_tile_block_mask),
 * §Recipe: STA with both repairs (evaluated at tile resolution it is the cluster-level
 * mask for tile_labels: expanding it through the labels reproduces the token-level
 * Sliding Tile Attention mask). Tiles of an nT x nH x nW tile grid in the raster order
 * of bsa_tile_labels; query tile a keeps key tile c when, on every axis, c lies in a's
 * window: the tiles within w/2 of a centre that is a moved inward at the borders
 * (clamped to [w/2, n-1-w/2]), so an odd window keeps w tiles; a window at least as
 * wide as the axis keeps all of them.
 *   wt, wh, ww : window sizes in tiles (>= 1).
 *   mask       : device uint8 (C, C), C = nT*nH*nW <= 16384; written (1 = kept).
 * Errors: INVALID_ARG for non-positive sizes or a null mask; UNSUPPORTED past 16384
 * tiles.
 */
int bsa_sliding_tile_block_mask(int nT, int nH, int nW, int wt, int wh, int ww, uint8_t* mask,
                                void* stream);

/*
 * antidiagonal_block_scores — [HMR] §XAttention — anti-diagonal block scoring,
 * §Deviations (rows normalised to 1), §Out of scope (the caller pads S to a multiple
 * of the block; padded keys take softmax mass).
 *   A[I,J] = sum_{t<s} q[I*s+t] . k[J*s+s-1-t]        (stride x stride anti-diagonals)
 *   P      = row-softmax(logit_scale * A) over all S/s columns
 *   scores[b,h,i,j] = (s/block) * sum over the (block/s)^2 entries of tile (i,j)
 * q: (B,Hq,S,D), k: (B,Hkv,S,D) with shape.Sq == shape.Sk == S; S % block == 0,
 * block % stride == 0, block/stride a power of two <= 32, S/stride a multiple of 128;
 * past S/stride = 2048 or S/block = 256 the GEMM runs twice (row statistics, then block
 * sums) and S/block >= 2 block/stride is needed; D in {64,128}; BSA_BF16 only (other sizes return
 * BSA_ERR_UNSUPPORTED). logit_scale <= 0 selects 1/sqrt(D).
 *   scores : device float32 (B, Hq, S/block, S/block), written; each row sums to 1.
 * The strided logit matrix is never written to device memory. No workspace.
 */
int bsa_antidiagonal_block_scores(const void* q, const void* k, bsa_shape shape, int block,
                                  int stride, float logit_scale, float* scores, void* stream);

/*
 * top_p_block_mask — [HMR] §XAttention (each query block keeps the smallest set of
 * key blocks whose mass reaches a fraction tau of its total), §Deviations (at least
 * one block per row; key block 0 not forced), §What mlx-arsenal ships (scalar or
 * per-head tau).
 * Per row: sort scores descending (equal scores: lower key index first), take the
 * running float32 sum in that order, keep ranks 0..m with m the first rank whose
 * running sum >= tau[h]; if no running sum reaches tau the whole row is kept.
 *   scores   : device float32 (B, H, Nq, Nk), Nk <= 1024.
 *   tau      : device float32, n_tau == 1 (shared) or n_tau == H (per head).
 *   mask     : device uint8 (B, H, Nq, Nk), written (1 = kept).
 *   tie_rows : device uint8 (B, H, Nq) or NULL; 1 where a running sum lies within
 *              1e-5 of tau or the last kept and first dropped scores differ by at most
 *              1e-5 (rows whose decision a different rounding could flip).
 */
int bsa_top_p_block_mask(const float* scores, int B, int H, int Nq, int Nk, const float* tau,
                         int n_tau, uint8_t* mask, uint8_t* tie_rows, void* stream);

/*
 * centroid_compensated_attention — [SBC] §The problem (block-sparse attention over
 * query/key clusters), §SVG-EAR — centroid compensation (every skipped key cluster c
 * enters the same softmax as ONE term with logit scale*q.kbar_c + ln n_c and value
 * vbar_c), §No LSE needed (equivalently one softmax over [K; Kbar]); [SPR] (Q, K, V
 * permuted into group-major order; hard drop renormalises over kept keys).
 *   q_labels : device int32 (Sq), values in [0, Cq).   k_labels: device int32 (Sk),
 *              values in [0, Ck). Labels outside the range make the output undefined.
 *   block_mask : device uint8 with element (b,h,a,c) at
 *              b*mask_b_stride + h*mask_h_stride + a*Ck + c; a stride of 0
 *              broadcasts (one mask for every batch and/or head).
 *   scale    : logit scale, <= 0 selects 1/sqrt(D).
 *   compensate : 1 = SVG-EAR compensation of skipped non-empty clusters;
 *              0 = hard drop (a row with no kept key outputs 0).
 *   out      : device float32 (B, Hq, Sq, D), written in original token order.
 *   workspace: >= bsa_attention_workspace_bytes(shape, Cq, Ck) bytes.
 * Centroids are arithmetic means per (batch, KV head, cluster), computed in fp32 and
 * rounded to the MMA input type. Limits: D in {64,128}; Ck <= 16384; Cq <= 16384;
 * Sk + 15*Ck <= 2^20 - 128 (key sequences longer than one CTA's window of 4096 key
 * groups are split into key ranges whose partial results are merged); B*Hq*Sq*16 and
 * B*Hkv*(Sk + 15*Ck) below 2^31. BSA_F32 inputs are computed with kind::tf32 MMAs.
 */
size_t bsa_attention_workspace_bytes(bsa_shape shape, int Cq, int Ck);
int bsa_centroid_compensated_attention(const void* q, const void* k, const void* v,
                                       bsa_shape shape, const int32_t* q_labels, int Cq,
                                       const int32_t* k_labels, int Ck,
                                       const uint8_t* block_mask, int64_t mask_b_stride,
                                       int64_t mask_h_stride, float scale, int compensate,
                                       float* out, void* workspace, size_t workspace_bytes,
                                       void* stream);

/*
 * centroid_compensated_attention_ex — the same call with flags. [HMR] §HEART and
 * "Reuse needs a fixed token grid" (labels fixed by the grid; masks reused across
 * denoising steps while the mask cache refreshes no head).
 *   flags & BSA_REUSE_PLAN : the workspace holds the preparation of an earlier call on
 *              it (label sorts, key cluster order, query tile plan, mask bitsets) with
 *              the same shape, q_labels, Cq, k_labels, Ck, block_mask contents and
 *              strides; those steps are skipped and the labels are not checked again.
 *              The K/V gather, the centroids and the attention run as usual, so q, k, v
 *              and scale may change between the calls. The caller owns that
 *              precondition: if the workspace does not hold such a preparation (or
 *              another call used it in between) the behaviour is undefined, and the
 *              kernels may read and write out of bounds. The Python binding passes the
 *              flag only for a workspace whose last attention call it recorded with
 *              the same arguments and unmodified label and mask tensors.
 * Other flag bits: BSA_ERR_INVALID_ARG. Arguments otherwise as
 * centroid_compensated_attention.
 */
int bsa_centroid_compensated_attention_ex(const void* q, const void* k, const void* v,
                                          bsa_shape shape, const int32_t* q_labels, int Cq,
                                          const int32_t* k_labels, int Ck,
                                          const uint8_t* block_mask, int64_t mask_b_stride,
                                          int64_t mask_h_stride, float scale, int compensate,
                                          float* out, void* workspace, size_t workspace_bytes,
                                          int flags, void* stream);

/*
 * per_kv_head_attention — the same attention with labels of their own per (batch, KV
 * head): [SPR] (K/V partitions and routes are shared by the query heads of a KV head;
 * the partition step produces one label set per KV head); [SBC] §Recipe (one
 * block-sparse call per label set).
 * For every (b, g) the G = Hq / Hkv query heads g*G .. g*G+G-1 attend to KV head g with
 * q_labels[b, g], k_labels[b, g] and mask slice (b, g):
 *   q_labels : device int32 (B, Hkv, Sq), values in [0, Cq).
 *   k_labels : device int32 (B, Hkv, Sk), values in [0, Ck).
 *   block_mask : device uint8, element (b, g, a, c) at b*mask_b_stride +
 *              g*mask_g_stride + a*Ck + c (a stride of 0 broadcasts).
 *   out      : device float32 (B, Hq, Sq, D), written in original token order.
 *   workspace: >= bsa_per_kv_head_attention_workspace_bytes(shape, Cq, Ck) bytes, used
 *              by the (b, g) problems one after another on the stream.
 * Other arguments, limits and errors as centroid_compensated_attention (the limits apply
 * to one (b, g) problem: B = Hkv = 1, Hq = G).
 */
size_t bsa_per_kv_head_attention_workspace_bytes(bsa_shape shape, int Cq, int Ck);
int bsa_per_kv_head_attention(const void* q, const void* k, const void* v, bsa_shape shape,
                              const int32_t* q_labels, int Cq, const int32_t* k_labels, int Ck,
                              const uint8_t* block_mask, int64_t mask_b_stride,
                              int64_t mask_g_stride, float scale, int compensate, float* out,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * error_aware_block_mask — SVG-EAR error-aware routing: [SBC] §SVG-EAR — centroid
 * compensation (an error-aware router chooses which blocks to compute exactly) and the
 * SVG-EAR abstract (a lightweight probe estimates each block's compensation error; the
 * blocks with the highest error-to-cost ratio are computed exactly, the rest
 * compensated). Per (b, query head h), with KV head h / (Hq / Hkv):
 *   probe of query cluster a : qbar_a, the mean query of the cluster;
 *   block error  err[a][c]   : || E - A ||_2 with, over the dense logits
 *                              l_j = scale qbar_a . k_j (max m, Z = sum_j exp(l_j - m)),
 *                              E = sum_{j in c} exp(l_j - m) v_j / Z (exact contribution)
 *                              A = n_c exp(scale qbar_a . kbar_c - m) vbar_c / Z (centroid);
 *   ratio                    : err[a][c] / n_c (error per computed pair), float32;
 *   mask[a][c] = 1           : the longest prefix of the blocks of non-empty clusters in
 *                              descending ratio (equal ratios: lower a*Ck + c) whose token
 *                              pairs n_a n_c sum to at most floor(density * Sq' * Sk'),
 *                              Sq', Sk' the rows with a valid label.
 *   q, k, v   : (B,Hq,Sq,D), (B,Hkv,Sk,D), (B,Hkv,Sk,D) device, BSA_BF16 or BSA_F32.
 *   q_labels  : device int32 (Sq) in [0, Cq);  k_labels : device int32 (Sk) in [0, Ck).
 *   density   : fraction of token pairs to compute exactly, in [0, 1].
 *   scale     : <= 0 selects 1/sqrt(D).
 *   mask      : device uint8 (B, Hq, Cq, Ck), written.
 *   err       : device float32 (B, Hq, Cq, Ck) or NULL; the block errors when given.
 *   workspace : >= bsa_routing_workspace_bytes(shape, Cq, Ck) bytes, 256-byte aligned.
 * Limits: D in {64,128}, Cq, Ck <= 16384, Cq*Ck <= 2^24. Errors: INVALID_ARG for null
 * pointers or a density outside [0, 1]; UNSUPPORTED past the limits; WORKSPACE.
 */
size_t bsa_routing_workspace_bytes(bsa_shape shape, int Cq, int Ck);
int bsa_error_aware_block_mask(const void* q, const void* k, const void* v, bsa_shape shape,
                               const int32_t* q_labels, int Cq, const int32_t* k_labels, int Ck,
                               float density, float scale, uint8_t* mask, float* err,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * probe_budget_block_mask — SparsePR's router with the probe cost reserved first: [SPR]
 * (executed-pair density is the routing density plus M/Nq; the router reserves the
 * probe cost first; whole cells are atomic). Per (b, query head), cells are scored by
 * their centroid-estimated attention mass: for the mean query qbar_a of query cluster a,
 *   mass[a][c] = softmax over non-empty key clusters of (scale qbar_a . kbar_c + ln n_c)
 * (0 for empty clusters), ranked by mass / n_c (mass per computed pair, equal ratios:
 * lower a*Ck + c), and the longest prefix whose pairs fit
 * floor(max(0, density - M / Sq) * Sq' * Sk') is kept (Sq', Sk' rows with a valid label).
 *   q, k      : (B,Hq,Sq,D), (B,Hkv,Sk,D) device, BSA_BF16 or BSA_F32.
 *   M         : probe rows reserved (>= 0).
 *   mask      : device uint8 (B, Hq, Cq, Ck), written. mass: float32 (B,Hq,Cq,Ck) or NULL.
 *   workspace : >= bsa_routing_workspace_bytes(shape, Cq, Ck) bytes, 256-byte aligned.
 * Limits and errors as error_aware_block_mask; INVALID_ARG for M < 0.
 */
int bsa_probe_budget_block_mask(const void* q, const void* k, bsa_shape shape,
                                const int32_t* q_labels, int Cq, const int32_t* k_labels, int Ck,
                                float density, int M, float scale, uint8_t* mask, float* mass,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * response_coupled_partition — SparsePR Response-Coupled Partitioning: [SPR] (queries
 * sampled from the call; keys grouped by their pre-softmax response, values following
 * their keys; key-group centroids define query coordinates so that queries with a
 * similar response direction share a route; one asymmetric pass; ranks rK = 48, rQ = 64;
 * K/V partitions and routes shared by a KV head's query heads; online k-means).
 * Per (b, KV head g), G = Hq / Hkv:
 *   samples      : rK query rows, sample s = token floor((s+1/2) Sq / rK) of query head
 *                  g*G + s % G;
 *   key features : f_j = scale * Q_s k_j (rK values per key), k-means into Ck groups;
 *   query coords : x_i = (scale * q_{h,i} . kbar_{c_t}) over rQ' = min(rQ, Ck) groups
 *                  c_t = floor((t+1/2) Ck / rQ') and the G heads, divided by its norm;
 *                  k-means into Cq groups.
 *   k-means      : Lloyd; centroids start at rows floor((c+1/2) N / C); `iters` rounds
 *                  of (nearest centroid by squared distance, ties to the lower index;
 *                  centroid = mean of its rows, an empty cluster keeps its centroid),
 *                  then a last assignment. Sums run in a fixed order (deterministic).
 *   q, k      : (B,Hq,Sq,D), (B,Hkv,Sk,D) device, BSA_BF16 or BSA_F32; D in {64,128}.
 *   q_labels  : device int32 (B, Hkv, Sq), written (one partition per KV head).
 *   k_labels  : device int32 (B, Hkv, Sk), written.
 *   scale     : <= 0 selects 1/sqrt(D).
 *   workspace : >= bsa_partition_workspace_bytes(shape, Cq, Ck, r_k, r_q), 256-aligned.
 * Limits: 1 <= Cq <= min(Sq, 4096), 1 <= Ck <= min(Sk, 4096), rK <= 256, rQ'*G <= 256.
 */
size_t bsa_partition_workspace_bytes(bsa_shape shape, int Cq, int Ck, int r_k, int r_q);
int bsa_response_coupled_partition(const void* q, const void* k, bsa_shape shape, int Cq, int Ck,
                                   int r_k, int r_q, int iters, float scale, int32_t* q_labels,
                                   int32_t* k_labels, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * select_probe_rows — [SBC] §What mlx-arsenal ships (round-robin over query clusters,
 * weights |G_a| / m_a), §Deviations (middle-out member; weights normalised to sum 1);
 * [SPR] (probes stratified across query groups and ordered by distance to the group
 * centroid).
 * Rows of each non-empty cluster are ranked: q == NULL -> middle-out (by
 * |r - (n-1)/2| of the row's rank r inside its cluster, ties to the lower rank),
 * shared by all heads; q != NULL -> per (batch, query head) by the Euclidean distance
 * to the cluster's mean query (ties to the lower index). With C' non-empty clusters,
 * M >= C' takes rank-p rows of every cluster in pass p until M rows are taken;
 * M < C' takes the first-ranked row of cluster floor(i*C'/M) for probe i.
 *   labels    : device int32 (S), values in [0, C).
 *   probe_idx : device int32 (M) if q == NULL, else (B, Hq, M); written.
 *   weights   : device float32, same shape; written, summing to 1 per head.
 *   shape     : used when q != NULL (B, Hq, Sq == S, D, dtype).
 * Limits: S <= 65536, C <= 16384, M <= 1024; with q, clusters of at most 4096 rows
 * (a larger cluster keeps index order and records BSA_ERR_UNSUPPORTED in the device
 * status). Workspace: bsa_probe_select_workspace_bytes(S, C, n_heads) with
 * n_heads = B*Hq when q != NULL, else 1.
 */
size_t bsa_probe_select_workspace_bytes(int S, int C, int n_heads);
int bsa_select_probe_rows(const int32_t* labels, int S, int C, int M, const void* q,
                          bsa_shape shape, int32_t* probe_idx, float* weights, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * probe_dense_attention — [SBC] §Recipe (exact attention of the probe rows over every
 * key); [SPR] (M query rows evaluated exactly against all keys).
 *   probe_idx : device int32 (M) shared (per_head == 0) or (B, Hq, M) (per_head == 1);
 *               an index outside [0, S) reads a zero row and records
 *               BSA_ERR_INVALID_ARG in the device status.
 *   o_probe   : device float32 (B, Hq, M, D), written.
 *   scale     : <= 0 selects 1/sqrt(D). M <= 1024. Workspace:
 *               bsa_probe_attention_workspace_bytes(shape, M).
 */
size_t bsa_probe_attention_workspace_bytes(bsa_shape shape, int M);
int bsa_probe_dense_attention(const void* q, const void* k, const void* v, bsa_shape shape,
                              const int32_t* probe_idx, int M, int per_head, float scale,
                              float* o_probe, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * probe_residual_correction — [SBC] §SparsePR — probe-fitted residual repair; [SPR]
 * (weighted ridge affine fit, lambda = 0.1, from the standardised sparse output,
 * projected on the top r = 16 residual directions, applied to all rows).
 * Per (b, h), with X = out[b,h] (S x D), Z = (X - mu) / sqrt(var + 1e-6) (column mean
 * and population variance over all S rows), Zt = [Z, 1], W = diag(weights):
 *   R    = o_probe - X[probe_idx]
 *   Bc   = (Zt_p^T W Zt_p + lam*diag(1,..,1,0))^-1 Zt_p^T W R   (Cholesky)
 *   V_r  = top-`rank` eigenvectors of R^T W R   (Householder, multisection, inverse iteration)
 *   out <- X + Zt * Bc * V_r V_r^T                                  (every row)
 *   out       : device float32 (B, H, S, D), updated in place.
 *   o_probe   : device float32 (B, H, M, D).
 *   probe_idx, weights : (M) shared (per_head == 0) or (B, H, M).
 * Limits: D in {64,128}, 1 <= rank <= D, M <= 1024. Workspace:
 * bsa_repair_workspace_bytes(B, H, S, D, M).
 */
size_t bsa_repair_workspace_bytes(int B, int H, int S, int D, int M);
int bsa_probe_residual_correction(float* out, const float* o_probe, const int32_t* probe_idx,
                                  const float* weights, int per_head, int B, int H, int S, int D,
                                  int M, int rank, float lam, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * probe_residual_correction_noalloc — no counterpart in the papers: a convenience for
 * callers that cannot allocate device memory when they repair an output (for example
 * a runtime whose device memory is fixed up front, or code on a path that must not
 * call the allocator). Same arguments and result as bsa_probe_residual_correction,
 * minus the workspace: the scratch comes from a 16 MiB buffer compiled into the
 * library, which every GPU that loads libbsa.so holds until the process exits.
 *  - Size limit: bsa_repair_workspace_bytes(B, H, S, D, M) must be <= 16 MiB (about
 *    B*H <= 48 heads at D = 128, M = 64); larger problems return BSA_ERR_UNSUPPORTED
 *    with the required size in the error detail.
 *  - The first call on each device looks up the buffer's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call before
 *    any stream capture begins.
 *  - Every call uses the same buffer: calls that may overlap on the GPU (different
 *    streams, or different host threads) race on it and must be serialised by the
 *    caller. The buffer needs no clearing; nothing is allocated or freed.
 */
int bsa_probe_residual_correction_noalloc(float* out, const float* o_probe,
                                          const int32_t* probe_idx, const float* weights,
                                          int per_head, int B, int H, int S, int D, int M,
                                          int rank, float lam, void* stream);

/*
 * Per-head drift/anchor mask cache — [HMR] §HEART — head-wise temporal mask reuse
 * (anchor = token means qbar, kbar and the head's mask; drift = L1 distance; refresh
 * above delta; layer gate: under gate_lo of the heads -> none, above gate_hi -> all),
 * §Deviations (relative drift divides by the anchor's L1 norm), §Recipe (every head
 * refreshes on the first call), "Reuse needs a fixed token grid" (reset on a grid
 * change).
 * State lives in a caller-owned device buffer of bsa_mask_cache_state_bytes() bytes;
 * it can be saved and restored like any tensor. One cache per layer and CFG branch.
 */
size_t bsa_mask_cache_state_bytes(int B, int H, int Cq, int Ck, int D);
/* Initialises the state (empty cache). gate_lo < 0 disables the layer gate. */
int bsa_mask_cache_init(void* state, int B, int H, int Cq, int Ck, int D, float delta,
                        int relative, float gate_lo, float gate_hi, void* stream);
/*
 * Pools q, k (B,H,S,D; Hkv must equal H) into per-head means, computes the drift
 * against the anchors, applies delta and the layer gate, and writes refresh
 * (device uint8 (B,H)). If n_refresh_host is non-NULL the stream is synchronised and
 * the number of refreshed heads is written there. drift_out (nullable) receives the
 * float32 (B,H) drift (+inf where no anchor exists yet). q and k must be 16-byte
 * aligned and D·(element size) a multiple of 16 bytes (D dividing 256), else
 * BSA_ERR_INVALID_ARG / BSA_ERR_UNSUPPORTED.
 */
int bsa_mask_cache_should_refresh(void* state, const void* q, const void* k, bsa_shape shape,
                                  uint8_t* refresh, float* drift_out, int* n_refresh_host,
                                  void* stream);
/*
 * Replaces the cached mask of every refreshed head by new_mask (device uint8
 * (B,H,Cq,Ck); may be NULL when no head refreshes), moves those heads' anchors to the
 * pooled values of the last should_refresh, and writes the resulting mask to
 * block_mask_out (device uint8 (B,H,Cq,Ck)).
 */
int bsa_mask_cache_update(void* state, const uint8_t* new_mask, const uint8_t* refresh,
                          uint8_t* block_mask_out, void* stream);
/*
 * Layer gate for a layer whose heads are split over several caches (one per GPU,
 * [HMR] §HEART: the gate looks at the fraction of the layer's heads asking for a
 * refresh). Each cache is initialised with gate_lo < 0 (no gate of its own); after
 * should_refresh the callers add their refresh counts over all GPUs (one integer
 * all-reduce) and pass the sum here: n_refresh_layer of n_heads_layer heads under
 * gate_lo -> none of this cache's heads refresh, above gate_hi -> all do, otherwise the
 * per-head flags stand. Not applied on a cache's first call. Updates `refresh` (device
 * uint8 (B, H) of this cache) in place. Errors: INVALID_ARG for null pointers or a
 * count outside [0, n_heads_layer].
 */
int bsa_mask_cache_layer_gate(void* state, uint8_t* refresh, int n_refresh_layer,
                              int n_heads_layer, float gate_lo, float gate_hi, void* stream);
/* Forgets anchors and masks: the next should_refresh refreshes every head. */
int bsa_mask_cache_reset(void* state, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H_ */
