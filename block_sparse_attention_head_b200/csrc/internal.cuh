// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace ig {

// ----------------------------------------------------------------- k-means
// Operand layout of the centroids for the tensor-core distance GEMM:
// [BH, c_pad, 2d] bf16, columns [0,d) = bf16(c) ("hi"), [d,2d) =
// bf16(c - hi) ("lo"); norm rows [BH, c_pad, kNormCols] bf16: -||c||^2 / 4
// of the fp32 centroid in three bf16 terms at columns 0-2 and again at 8-10,
// zeros elsewhere (padding rows: -inf at columns 0 and 8).  One more K = 16
// step of the distance MMA, against a block of ones at columns 0-2 and 8-10
// of every token row, adds -||c||^2 / 2 to x.c; the copies in both 16-byte
// halves keep that sum independent of where a swizzle puts the halves.
// Columns 16-31 are zeros (the hi | lo layout below takes them as the lo
// CTA's norm block).
constexpr int kNormCols = 32;
struct KmeansGeom {
  int BH, N, d, C;
  int chunk;   // centroids per MMA chunk (multiple of 16, <= 256)
  int c_pad;   // C rounded up to a multiple of chunk
};
KmeansGeom kmeans_geom(int BH, int N, int d, int C);
// One resident chunk of at most 128 centroids: the assign MMA takes the hi
// and lo operand halves side by side along N (N = 2 * chunk, K = d; one CTA of
// the pair holds the hi rows, the other the lo rows) instead of one after
// the other along K, which halves its MMA count.
__host__ __device__ inline bool kmeans_hilo_n(const KmeansGeom& g) { return g.c_pad == g.chunk && g.chunk <= 128; }

// The centroid update splits a cluster of n members into pieces of at most
// kUpdRows consecutive permuted rows (an empty cluster is one empty piece);
// its grid has kmeans_update_grid(g) CTAs per head, piece t of a head being
// entry t of the head's piece map, {cluster, piece, pieces of the cluster,
// first partial-sum slot of the cluster} ({-1, ...} past the last piece),
// which the counting sort of the same iteration writes.
constexpr int kUpdRows = 2048;
__host__ __device__ inline int update_pieces(int n) { return n <= kUpdRows ? 1 : (n + kUpdRows - 1) / kUpdRows; }
inline int kmeans_update_grid(const KmeansGeom& g) { return g.C + (g.N + kUpdRows - 1) / kUpdRows; }

// Scratch of one clustering call, carved from one 256-byte aligned block:
// the operand rows and norm rows above, the piece map above ([BH,
// kmeans_update_grid] int4), fp32 partial sums of the clusters that
// the update splits into several row pieces ([BH, part_slots, d]), and one
// arrival counter per (head, cluster) ([BH, C] int32, zeroed by the init
// kernel and returned to zero by the update that consumes it).
struct KmeansScratch {
  __nv_bfloat16* cmma;
  __nv_bfloat16* nrow;
  int4* pmap;
  float* partial;
  int32_t* arrive;
};
int kmeans_part_slots(const KmeansGeom& g);
size_t kmeans_scratch_bytes(const KmeansGeom& g);
KmeansScratch kmeans_scratch_carve(const KmeansGeom& g, void* ws);

cudaError_t launch_kmeans_init(const KmeansGeom& g, const __nv_bfloat16* X, const float* init, float* cent,
                               const KmeansScratch& sc, cudaStream_t s);
cudaError_t launch_kmeans_assign(const KmeansGeom& g, const CUtensorMap* tmap_x, const CUtensorMap* tmap_c,
                                 const CUtensorMap* tmap_n, int32_t* assign, cudaStream_t s);
cudaError_t launch_kmeans_update(const KmeansGeom& g, const __nv_bfloat16* X, const int32_t* perm,
                                 const int32_t* offsets, float* cent, const KmeansScratch& sc, cudaStream_t s);

// ------------------------------------------------------- permutation/gather
// pmap (may be null): the centroid update's piece map, written from the
// cluster sizes (kmeans_update_grid(geometry) entries per head).
cudaError_t launch_count_sort(const int32_t* assign, int BH, int N, int C, int32_t* perm, int32_t* offsets,
                              int4* pmap, int pgrid, cudaStream_t s);
// Up to two tensors gathered with the same permutation (X1 may be null); a
// tensor with its f16 flag set is converted bf16 -> fp16.
cudaError_t launch_gather_rows(const __nv_bfloat16* X0, const __nv_bfloat16* X1, const int32_t* perm, int BH,
                               int N, int d, void* Y0, void* Y1, bool f16_0, bool f16_1, cudaStream_t s);

// ---------------------------------------------------------- select/sample
struct SelectArgs {
  const float* cq;
  const float* ck;
  const int32_t* k_offsets;
  int BH, Cq, Ck, d;
  float scale;
  long long E, m;
  unsigned long long seed;
  unsigned layer;
  int mode;
  int bh0;  // global index of head 0 of this launch (the Philox counter's head)
  const int32_t* votes;  // [BH,Cq,Ck] product-quantised votes, or null (rank by S alone)
  int top_p;             // 1: top-p selection (rank by mass, keep a share p_fix / 2^20, no sample)
  long long p_fix;       // round(top_p * 2^20)
  long long floor_keys;  // least number of kept keys
  int32_t* exact_groups;
  int32_t* counts;
  int32_t* sample_pos;
  float* sample_bias;
};
cudaError_t launch_select_sample(const SelectArgs& a, cudaStream_t s);

// ------------------------------------------------- product-quantised votes
struct PqArgs {
  const float* cq;                  // [BH,Cq,d] query group centroids
  const float* ck;                  // [BH,Ck,d] key group centroids
  const __nv_bfloat16* Q;           // [BH,N,d] original order
  const int32_t* q_perm;            // [BH,N]
  const int32_t* q_offsets;         // [BH,Cq+1]
  const int32_t* k_offsets;         // [BH,Ck+1]
  int BH, N, d, Cq, Ck;
  long long E;                      // exact-key budget
  float* codebooks;                 // [BH][2][d/8][16][8] (set by launch_pq_votes)
  uint8_t* kcodes;                  // [BH][Ck][d/8] (set by launch_pq_votes)
  int32_t* votes;                   // [BH,Cq,Ck]
};
size_t pq_scratch_bytes(int BH, int d, int Ck);
cudaError_t launch_pq_votes(const PqArgs& a, void* scratch, cudaStream_t s);

// --------------------------------------------------------------- attention
struct AttnArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* Kp;
  const __half* Vp;  // fp16 (converted by the gather)
  const int32_t* q_perm;
  const int32_t* q_offsets;
  const int32_t* k_offsets;
  const int32_t* exact_groups;
  const int32_t* counts;
  const int32_t* sample_pos;
  const float* sample_bias;
  __nv_bfloat16* O;
  int BH, N, d, Cq, Ck;
  long long m;
  float scale_log2;  // softmax_scale * log2(e)
};
constexpr int kAttnMaxExactGroups = 2048;
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s);

// ------------------------------------------------------------------ errors
cudaError_t read_and_clear_device_error(int* value, cudaStream_t s);

}  // namespace ig
