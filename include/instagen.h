/*
 * instagen.h -- C ABI of libinstagen.so: InstaGen group-shared importance-
 * sampled permuted block-sparse attention (PBSA) for one DiT self-attention
 * call, on one NVIDIA B200 (sm_100a).
 *
 * Method (InstaGen: Group-Shared Importance Sampling for Fast Video
 * Generation, arXiv 2611.08610; abstract, and Figure 3 (a)-(d) of the
 * thelatestinai.com paper page).  Per head:
 *   (a) k-means splits the queries into Cq groups and the keys into Ck
 *       groups, and a permutation makes every group a contiguous block;
 *   (b) from centroid scores each query group gets a probability pi over
 *       the key groups;
 *   (c) the best-ranked key groups make up an exact set (never empty: the
 *       first-ranked group is in it); the remaining keys are covered by m
 *       draws in proportion to pi,
 *       one list shared by every query of the group, each draw carrying the
 *       log-weight log(1/(pi*m));
 *   (d) exact blocks and sampled keys go through one online-softmax kernel.
 *
 * Conventions shared by every entry point
 *   - Tensors are contiguous, row-major, on the current CUDA device.
 *     Q, K, V, O: [B, H, N, d] bf16.  B and H are folded: head bh = b*H + h.
 *   - Device pointers unless stated.  The caller owns every buffer; the
 *     library never allocates or frees memory and never synchronises
 *     (except instagen_device_status, which synchronises the given stream).
 *     instagen_forward_host alone creates helper streams and events, and
 *     releases them before it returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     All work is enqueued asynchronously on it.
 *   - Return value: an instagen_status.  Argument errors are detected on the
 *     host before anything is enqueued.  Kernels never trap: an index found
 *     out of range on the device is skipped and recorded, and a wait that
 *     exceeds its bound aborts the kernel; both are reported by
 *     instagen_device_status.
 *   - Permuted order: cluster c of a head occupies permuted slots
 *     [offsets[c], offsets[c+1]); perm[p] is the original token index at slot
 *     p.  Inside a cluster tokens keep ascending original index.
 */
#ifndef INSTAGEN_H
#define INSTAGEN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IG_OK = 0,
  IG_ERR_INVALID_ARG = 1,   /* bad pointer, shape, or parameter value            */
  IG_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. d not in {64, 128})     */
  IG_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required        */
  IG_ERR_CUDA = 4,          /* a CUDA runtime call failed                         */
  IG_ERR_DEVICE_CHECK = 5   /* a kernel recorded an out-of-range index / timeout */
} instagen_status;

typedef enum { IG_SAMPLE_IMPORTANCE = 0, IG_SAMPLE_UNIFORM = 1 } instagen_sampling;
/* How the exact set is ranked: by centroid scores (Figure 3 (b)-(c)), by
 * product-quantised per-query votes (the abstract's rule; see
 * instagen_pq_votes), or by the top-p rule of the comparator the pages set
 * InstaGen against (thelatestinai.com paper page, Figure 2 caption: SVG2 at
 * top-p 0.5 to 0.95 with key floor 0.1; ICLR listing abstract: top-p keeps
 * the best blocks until a target share of the attention mass is reached and
 * skips the rest).  Top-p: key group j's estimated mass is |K_j| q_j (the
 * sampler's integer weights, taken over every non-empty group), groups are
 * kept in descending mass order (ties: lower j) until their share of the
 * total reaches top_p (compared in integers as cum * 2^20 >= round(top_p *
 * 2^20) * total) and at least round(key_floor * N) keys are kept; the
 * first-ranked group is always kept; there is no sample (sample_frac must
 * give m = 0) and exact_frac is unused. */
typedef enum { IG_SELECT_CENTROID = 0, IG_SELECT_PQ_VOTE = 1, IG_SELECT_TOP_P = 2 } instagen_selection;

typedef struct {
  int32_t B, H, N, d;        /* shapes; d in {64, 128}; N >= 1                     */
  int32_t Cq, Ck;            /* query / key cluster counts (Figure 2: 100 / 500)    */
  int32_t kmeans_iters;      /* Lloyd iterations (>= 1; 10 in every configuration) */
  float exact_frac;          /* exact share of keys: E = round(exact_frac * N)      */
  float sample_frac;         /* sampled share: m = round(sample_frac * N) draws      */
  float softmax_scale;       /* logit scale > 0, usually 1/sqrt(d)                   */
  uint64_t seed;             /* Philox key                                           */
  uint32_t layer;            /* Philox counter word 3 (one stream per layer)         */
  int32_t sampling;          /* instagen_sampling                                    */
  int32_t selection;         /* instagen_selection (PQ voting, top-p: N < 2^20)     */
  float top_p;               /* top-p selection: mass share in [0, 1]                */
  float key_floor;           /* top-p selection: least share of keys kept, in [0, 1] */
} instagen_params;

/* E and m for these parameters: the share times N rounded to nearest, halves
 * away from zero (Table 1 caption: E + S denotes the fraction of keys attended
 * exactly plus the fraction sampled, per sparse call). */
int64_t instagen_exact_budget(const instagen_params* p);
int64_t instagen_sample_budget(const instagen_params* p);

/* Workspace bytes instagen_forward needs for these parameters (0 if invalid).
 * Other entry points document their own needs. */
size_t instagen_workspace_size(const instagen_params* p);

/* Workspace bytes instagen_cluster needs for C clusters. */
size_t instagen_cluster_workspace_size(const instagen_params* p, int32_t C);

/* Human-readable text for a status code (static storage). */
const char* instagen_error_string(int status);

/* Synchronises `stream`, then returns IG_ERR_DEVICE_CHECK and clears the
 * device error word if any kernel of this library recorded an out-of-range
 * index or a wait timeout since the last call; IG_OK otherwise. */
int instagen_device_status(void* stream);

/*
 * (a) k-means clustering + stable permutation of one tensor X (Q or K),
 *     Figure 3 (a); the abstract's reordering of tokens by cluster.
 *   X         [B,H,N,d] bf16.
 *   C         cluster count, 1 <= C <= 4096.
 *   iters     Lloyd iterations >= 1 (each: assign to the nearest centroid by
 *             squared Euclidean distance, lowest index on ties; then every
 *             non-empty cluster's centroid becomes its members' mean, an empty
 *             cluster keeps its centroid).
 *   init      [B,H,C,d] fp32 initial centroids, or NULL for centroid j =
 *             token floor(j*N/C) of the head.
 *   centroids [B,H,C,d] fp32 out: centroids after the last update (the means
 *             of the returned clusters).
 *   assign    [B,H,N] int32 out: cluster of every token (last iteration).
 *   perm      [B,H,N] int32 out; offsets [B,H,C+1] int32 out (see above).
 *   ws        >= instagen_cluster_workspace_size(p, C) bytes, 256-B aligned.
 * Distances are evaluated on the tensor cores as ||c||^2 - 2 x.c (the argmax
 * of x.c - ||c||^2 / 2) with the fp32 centroid split into two bf16 halves (hi +
 * lo), ||c||^2 / 2 in three bf16 terms, and fp32 accumulation.
 */
int instagen_cluster(const void* X, int32_t C, int32_t iters, const float* init, const instagen_params* p,
                     float* centroids, int32_t* assign, int32_t* perm, int32_t* offsets, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * instagen_cluster without a workspace argument: the same k-means +
 * permutation, with its scratch (centroid operand and norm rows, the update's
 * piece map, partial sums
 * and arrival counters of the centroid update) in a device
 * array of INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES that the library itself
 * owns.  No counterpart on the method's pages; this exists for callers that
 * may not allocate device memory themselves -- plug-ins inside a host
 * framework whose allocator owns all device memory, deployments that fix
 * their memory budget at start-up and forbid later allocations, and code
 * paths where a cudaMalloc would implicitly synchronise the device.
 *   Arguments and outputs as instagen_cluster.  Nothing is allocated: no
 *   cudaMalloc, cudaFree or allocating library routine is called.
 *   Scratch needed = instagen_cluster_workspace_size(p, C); larger requests
 *   return IG_ERR_WORKSPACE before anything is enqueued.  The scratch grows
 *   with B*H, C and d, and a little with N (8*d bytes per 2048 tokens of a
 *   head): 16 MiB covers up to 48 heads at C <= 512, d = 128, N = 75600
 *   (e.g. the 40-head key clustering of Wan2.1-14B at 720p).
 *   The array is held by every GPU that loads the library until the process
 *   exits.  The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  The address is looked up again when the
 *   device's current context changes (after cudaDeviceReset, for instance),
 *   so the first call after such a change must also come before any capture.
 *   All calls share the one array and it keeps the last call's contents;
 *   every element a call reads is written by the same call first, so nothing
 *   needs clearing, but calls that overlap on the GPU (other streams, other
 *   threads) race on it: serialise them.
 */
#define INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
int instagen_cluster_static(const void* X, int32_t C, int32_t iters, const float* init, const instagen_params* p,
                            float* centroids, int32_t* assign, int32_t* perm, int32_t* offsets, void* stream);

/*
 * Stable counting sort of given assignments (the permutation step alone).
 *   assign [B,H,N] int32 in [0, C); perm [B,H,N] out; offsets [B,H,C+1] out.
 * Out-of-range assignments are an IG_ERR_DEVICE_CHECK (the token is dropped).
 */
int instagen_permutation(const int32_t* assign, int32_t C, const instagen_params* p, int32_t* perm,
                         int32_t* offsets, void* stream);

/*
 * Gather rows into permuted order: Xp[bh, s, :] = X[bh, perm[bh, s], :].
 *   X [B,H,N,d] bf16; perm [B,H,N] int32; Xp [B,H,N,d] (distinct buffer):
 *   bf16 when to_f16 = 0 (keys), fp16 when to_f16 = 1 (values: the attention
 *   kernel multiplies fp16 P by fp16 V).  Values beyond the fp16 range are
 *   saturated to +-65504 and reported as IG_ERR_DEVICE_CHECK.
 */
int instagen_gather(const void* X, const int32_t* perm, const instagen_params* p, void* Xp, int32_t to_f16,
                    void* stream);

/*
 * (b)+(c) Centroid scores, exact set and the group-shared sample
 *   (abstract: the highest-scoring keys are attended exactly and the others
 *   through a sample drawn with probability following their estimated
 *   attention, weighted by the inverse of that probability; Figure 3 (b),
 *   (c)).
 *   cq [B,H,Cq,d] fp32, ck [B,H,Ck,d] fp32 centroids (ck 16-byte aligned);
 *   k_offsets [B,H,Ck+1].
 *   Score S_ij = fp32 fused-multiply-add chain of cq_i . ck_j over k = 0..d-1,
 *   then one fp32 multiply by softmax_scale (bit-reproducible).
 *   Exact set of query group i: non-empty key groups ranked by S_ij descending
 *   (ties: lower j first); rank 0 always; then while the key count stays <= E.
 *   pi: key k of skipped group j has probability q_j / T, q_j in [1, 2^24] the
 *   integer 2^24 * exp(S_ij - max skipped S) (uniform mode: q_j = 1), T = sum
 *   over skipped groups of |K_j| q_j.  Draw t of group i: Philox4x32-10 with
 *   key (seed low, seed high) and counter (t, i, bh, layer); u = r1*2^32 + r0;
 *   r = floor(u*T / 2^64); group = first j (ascending) whose inclusive CDF
 *   exceeds r; key = offsets[j] + (r - CDF_{j-1}) / q_j.  Log-weight
 *   ln T - ln q_j - ln m (fp32).  No skipped keys: no draws.
 * Outputs (per head, per query group i):
 *   exact_groups [B,H,Cq,Ck] int32: exact groups in rank order, then -1.
 *   counts       [B,H,Cq,3] int32: {exact groups, exact keys, draws}.
 *   sample_pos   [B,H,Cq,m] int32: permuted key slots in draw order (-1 unused).
 *   sample_bias  [B,H,Cq,m] fp32 log-weights (0 unused).
 *   m = instagen_sample_budget(p); sample_pos/sample_bias may be NULL if m = 0.
 *   Requires Ck <= 4096.
 */
/*
 * Product-quantised per-query voting (abstract: queries and keys are product-
 * quantised so a block score is cheap for every query, not only for the
 * cluster centroid; each query votes for its top blocks; the cluster attends
 * to the blocks with the most votes).  The pages fix nothing further; read
 * here as: subspaces of 8 consecutive dimensions (M = d/8), 16 codewords per
 * subspace and side, trained per head by 5 Lloyd iterations on that side's
 * group centroids (start: the first min(16, C) centroids; squared distances
 * as an fma chain of the 8 differences; ties to the lowest codeword; update
 * = fp32 sum of the members in point order / their count; empty codewords
 * keep their value); query tokens encoded against the query codebook, key
 * groups by their centroids against the key codebook; block score = sum over
 * m ascending (fp32 from +0) of T_m[a_m(q)][b_m(j)], T_m = fma-chain inner
 * products of the two codebooks' codewords; query q votes for the prefix of
 * its ranking (non-empty groups by score descending, ties lower j) that the
 * exact-set budget rule takes (rank 0 always, then while the key count stays
 * <= E).  Every decision is a correctly rounded fp32 step in a fixed order.
 *   Q [B,H,N,d] bf16 original order; cq, ck, q_perm, q_offsets, k_offsets as
 *   produced by instagen_cluster; votes [B,H,Cq,Ck] int32 (out).
 *   ws: device scratch of instagen_pq_votes_workspace_size(p) bytes, 256-byte
 *   aligned (codebooks and key-group codes).  Requires N < 2^20.
 */
size_t instagen_pq_votes_workspace_size(const instagen_params* p);
int instagen_pq_votes(const void* Q, const float* cq, const float* ck, const int32_t* q_perm,
                      const int32_t* q_offsets, const int32_t* k_offsets, const instagen_params* p, int32_t* votes,
                      void* ws, size_t ws_bytes, void* stream);

/* instagen_select_sample with the exact set ranked by votes [B,H,Cq,Ck]
 * (descending; saturated at 2^20 - 1) before S_ij and j; pi and the sample
 * as in instagen_select_sample. */
int instagen_select_sample_votes(const float* cq, const float* ck, const int32_t* k_offsets, const int32_t* votes,
                                 const instagen_params* p, int32_t* exact_groups, int32_t* counts,
                                 int32_t* sample_pos, float* sample_bias, void* stream);

int instagen_select_sample(const float* cq, const float* ck, const int32_t* k_offsets, const instagen_params* p,
                           int32_t* exact_groups, int32_t* counts, int32_t* sample_pos, float* sample_bias,
                           void* stream);

/*
 * (d) Sparse attention over exact blocks plus the weighted sample, one
 *   online-softmax pass (Figure 3 (d); ICLR listing abstract: the sampled keys
 *   and the top-k blocks are processed by the same attention kernel).
 *   Q  [B,H,N,d] bf16 in ORIGINAL token order (rows gathered via q_perm).
 *   Kp [B,H,N,d] bf16 and Vp [B,H,N,d] fp16, both in key-cluster (permuted)
 *   order (instagen_gather with to_f16 = 0 and 1).
 *   q_perm, q_offsets: query permutation; k_offsets: key cluster ranges.
 *   exact_groups, counts, sample_pos, sample_bias: as instagen_select_sample.
 *   O  [B,H,N,d] bf16 out, ORIGINAL token order.  Query q of group i gets
 *   softmax over {scale*q.k : k in exact groups of i} U {scale*q.k_t + bias_t :
 *   sample slots t of i} applied to the matching V rows (a key drawn twice
 *   counts twice).
 * QK^T runs on the tcgen05 tensor cores with bf16 operands and PV with fp16
 * operands (P = exp2 of the shifted logits, <= 256, rounded to fp16), both
 * accumulating in fp32 in TMEM; O is rounded to bf16 once at the end.
 */
int instagen_attention(const void* Q, const void* Kp, const void* Vp, const int32_t* q_perm,
                       const int32_t* q_offsets, const int32_t* k_offsets, const int32_t* exact_groups,
                       const int32_t* counts, const int32_t* sample_pos, const float* sample_bias,
                       const instagen_params* p, void* O, void* stream);

/*
 * The whole call: cluster Q (Cq) and K (Ck), gather K and V into key-cluster
 * order, select and sample, attend.  O [B,H,N,d] bf16 in original order.
 * ws >= instagen_workspace_size(p) bytes, 256-B aligned; it holds every
 * intermediate (layout: instagen_forward_layout).
 */
int instagen_forward(const void* Q, const void* K, const void* V, void* O, const instagen_params* p, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * instagen_forward with initial centroids for both clusterings (a warm
 * start, e.g. from the previous denoising step's centroids, run with fewer
 * k-means iterations).  No separate counterpart on the pages; it serves the
 * step-to-step reuse of the clustering that the pages' warm-up/step
 * structure invites.  cq_init [B,H,Cq,d] and ck_init [B,H,Ck,d] fp32 device
 * pointers, each may be NULL (that clustering starts from tokens
 * floor(j*N/C)).  They may point at the cq / ck blocks of the same workspace
 * (instagen_forward_layout: the previous call's final centroids): each row
 * is read before it is overwritten.  Otherwise as instagen_forward.
 */
int instagen_forward_init(const void* Q, const void* K, const void* V, void* O, const instagen_params* p,
                          const float* cq_init, const float* ck_init, void* ws, size_t ws_bytes, void* stream);

/*
 * instagen_forward with HOST buffers: Q, K, V (inputs) and O (output) are
 * host memory in the [B,H,N,d] bf16 layout of instagen_forward.  No
 * counterpart on the method's pages: the heads are independent, so the call
 * splits them into chunks of at most heads_per_chunk consecutive heads of
 * one batch row (0: chosen by the library, about 160 MB per tensor per
 * chunk) and pipelines them: while chunk c is computed, the next chunks are
 * copied in on one copy stream and chunk c - 1 copied out on another, so the
 * PCIe transfers overlap the kernels.  A row's first chunk is one head (the
 * kernels start after one head's copy), each next chunk half again as large
 * as the one before up to heads_per_chunk (its copy in then ends before the
 * chunk in front of it is computed), and its last chunk one head (a short
 * drain).  A chunk's Q, K and V are copied in that order and its kernels
 * start once its Q is in.  The result equals instagen_forward on
 * device copies of the same inputs, bit for bit (every head draws its sample
 * with its global head index).
 *   Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister);
 *   pageable memory works but the copies then do not overlap.
 *   ws >= instagen_forward_host_workspace_size(p, heads_per_chunk) bytes of
 *   DEVICE memory, 256-B aligned: three staging slots, each a chunk's Q, K,
 *   V and O plus one of instagen_forward's workspaces for one chunk
 *   (consecutive chunks run on two compute streams, `stream` and an internal
 *   one, so one chunk's last kernels overlap the next chunk's first).
 *   Everything is enqueued asynchronously; `stream` is ordered after all of
 *   it (synchronise it before reading O).  The internal streams and their
 *   events are created and released inside the call, so it must not run
 *   during stream capture.  Overlapping calls that share `ws` race.
 */
size_t instagen_forward_host_workspace_size(const instagen_params* p, int32_t heads_per_chunk);
int instagen_forward_host(const void* Q, const void* K, const void* V, void* O, const instagen_params* p,
                          int32_t heads_per_chunk, void* ws, size_t ws_bytes, void* stream);

/* Byte offsets of instagen_forward's intermediates inside its workspace, so a
 * caller can inspect them after a call (every offset is 256-B aligned). */
typedef struct {
  size_t cq, ck;                 /* fp32 centroids [B,H,Cq,d], [B,H,Ck,d]      */
  size_t q_assign, k_assign;     /* int32 [B,H,N]                               */
  size_t q_perm, k_perm;         /* int32 [B,H,N]                               */
  size_t q_offsets, k_offsets;   /* int32 [B,H,Cq+1], [B,H,Ck+1]                */
  size_t kp, vp;                 /* [B,H,N,d] permuted K (bf16) and V (fp16)    */
  size_t exact_groups, counts;   /* int32 [B,H,Cq,Ck], [B,H,Cq,3]               */
  size_t sample_pos, sample_bias;/* int32 / fp32 [B,H,Cq,m]                     */
  size_t votes, pq_ws;           /* PQ voting: int32 [B,H,Cq,Ck] and its scratch
                                    (0 bytes unless selection = PQ voting)     */
  size_t cluster_ws;             /* scratch for instagen_cluster                */
  size_t total;                  /* == instagen_workspace_size                  */
} instagen_forward_layout;

int instagen_forward_layout_get(const instagen_params* p, instagen_forward_layout* out);

#ifdef __cplusplus
}
#endif

#endif /* INSTAGEN_H */
