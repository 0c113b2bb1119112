// C ABI of libinstagen.so (declared in include/instagen.h): argument checks,
// workspace carving, TMA descriptor setup and the launch sequence of the
// InstaGen attention call (cluster -> permute/gather -> select/sample ->
// attend).  Nothing here computes on the host beyond shapes and budgets.
#include "instagen.h"
#include "internal.cuh"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

namespace {

using ig::KmeansGeom;

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and parameter checks shared by every entry point.
int check_params(const instagen_params* p) {
  if (!p) return IG_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1) return IG_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return IG_ERR_UNSUPPORTED;
  const long long bh = (long long)p->B * p->H;
  if (bh > 65535) return IG_ERR_UNSUPPORTED;                       // grid.y
  if (bh * (long long)p->N > 2147483647LL - 1024) return IG_ERR_UNSUPPORTED;  // int32 row indices
  if (!std::isfinite(p->exact_frac) || !std::isfinite(p->sample_frac) || p->exact_frac < 0.f ||
      p->sample_frac < 0.f)
    return IG_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale) || !(p->softmax_scale > 0.f)) return IG_ERR_INVALID_ARG;
  if (p->sampling != IG_SAMPLE_IMPORTANCE && p->sampling != IG_SAMPLE_UNIFORM) return IG_ERR_INVALID_ARG;
  if (p->selection != IG_SELECT_CENTROID && p->selection != IG_SELECT_PQ_VOTE && p->selection != IG_SELECT_TOP_P)
    return IG_ERR_INVALID_ARG;
  // votes enter the rank key saturated at 2^20 - 1: a group has fewer queries;
  // top-p compares masses (< N * 2^24) scaled by 2^20 in 64 bits
  if ((p->selection == IG_SELECT_PQ_VOTE || p->selection == IG_SELECT_TOP_P) && p->N > 0xFFFFF)
    return IG_ERR_UNSUPPORTED;
  if (p->selection == IG_SELECT_TOP_P) {
    if (!(p->top_p >= 0.f && p->top_p <= 1.f) || !(p->key_floor >= 0.f && p->key_floor <= 1.f))
      return IG_ERR_INVALID_ARG;
    if (llround((double)p->sample_frac * (double)p->N) != 0) return IG_ERR_INVALID_ARG;  // no sample
  }
  return IG_OK;
}

int check_clusters(int C) {
  if (C < 1) return IG_ERR_INVALID_ARG;
  if (C > 4096) return IG_ERR_UNSUPPORTED;
  return IG_OK;
}

long long budget(float frac, int N) { return (long long)llround((double)frac * (double)N); }

int check_budgets(const instagen_params* p) {
  const long long m = budget(p->sample_frac, p->N);
  const long long E = budget(p->exact_frac, p->N);
  if (m > 2147483647LL || E > 2147483647LL) return IG_ERR_UNSUPPORTED;
  if ((long long)p->B * p->H * p->Cq * (m > 0 ? m : 1) > (1LL << 40)) return IG_ERR_UNSUPPORTED;
  return IG_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? IG_OK : IG_ERR_CUDA; }

// ------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] tensor, box {64 columns, box_rows rows},
// 128-byte swizzle (the UMMA K-major SWIZZLE_128B layout), zero fill outside;
// or (box_cols 16) box {16 columns, box_rows rows} with the 32-byte swizzle of
// the UMMA K-major SWIZZLE_32B layout.
int make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                   uint32_t box_cols = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return IG_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IG_OK : IG_ERR_CUDA;
}

// ---------------------------------------------------------------- cluster
int run_cluster(const void* X, int C, int iters, const float* init, const instagen_params* p, float* cent,
                int32_t* assign, int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes, cudaStream_t s) {
  const int BH = p->B * p->H;
  const KmeansGeom g = ig::kmeans_geom(BH, p->N, p->d, C);
  if (!ws || ws_bytes < ig::kmeans_scratch_bytes(g) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return IG_ERR_WORKSPACE;
  const ig::KmeansScratch sc = ig::kmeans_scratch_carve(g, ws);
  CUtensorMap tx, tc, tn;
  int rc = make_tmap_bf16(&tx, X, (uint64_t)BH * p->N, (uint64_t)p->d, 128);
  if (rc) return rc;
  // centroid operand boxes: half a chunk per CTA, or (hi | lo along N) the
  // whole chunk, hi columns in one CTA and lo in the other
  rc = make_tmap_bf16(&tc, sc.cmma, (uint64_t)BH * g.c_pad, (uint64_t)2 * p->d,
                      (uint32_t)(ig::kmeans_hilo_n(g) ? g.chunk : g.chunk / 2));
  if (rc) return rc;
  // norm rows: the same rows per CTA, 16 columns (hi | lo: the lo CTA takes
  // the zero columns 16-31)
  rc = make_tmap_bf16(&tn, sc.nrow, (uint64_t)BH * g.c_pad, (uint64_t)ig::kNormCols,
                      (uint32_t)(ig::kmeans_hilo_n(g) ? g.chunk : g.chunk / 2), 16);
  if (rc) return rc;
  const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
  cudaError_t e = ig::launch_kmeans_init(g, Xb, init, cent, sc, s);
  for (int it = 0; it < iters && e == cudaSuccess; ++it) {
    e = ig::launch_kmeans_assign(g, &tx, &tc, &tn, assign, s);
    if (e == cudaSuccess)
      e = ig::launch_count_sort(assign, BH, p->N, C, perm, offsets, sc.pmap, ig::kmeans_update_grid(g), s);
    if (e == cudaSuccess) e = ig::launch_kmeans_update(g, Xb, perm, offsets, cent, sc, s);
  }
  return cuda_status(e);
}

struct ForwardLayout {
  instagen_forward_layout l;
};

int forward_layout(const instagen_params* p, instagen_forward_layout* L) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(p->Cq)) || (rc = check_clusters(p->Ck))) return rc;
  if ((rc = check_budgets(p))) return rc;
  const size_t BH = (size_t)p->B * p->H, N = p->N, d = p->d;
  const size_t m = (size_t)budget(p->sample_frac, p->N);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L->cq = take(BH * p->Cq * d * 4);
  L->ck = take(BH * p->Ck * d * 4);
  L->q_assign = take(BH * N * 4);
  L->k_assign = take(BH * N * 4);
  L->q_perm = take(BH * N * 4);
  L->k_perm = take(BH * N * 4);
  L->q_offsets = take(BH * (p->Cq + 1) * 4);
  L->k_offsets = take(BH * (p->Ck + 1) * 4);
  L->kp = take(BH * N * d * 2);
  L->vp = take(BH * N * d * 2);
  L->exact_groups = take(BH * p->Cq * p->Ck * 4);
  L->counts = take(BH * p->Cq * 3 * 4);
  L->sample_pos = take(BH * p->Cq * (m ? m : 1) * 4);
  L->sample_bias = take(BH * p->Cq * (m ? m : 1) * 4);
  const bool pq = p->selection == IG_SELECT_PQ_VOTE;
  L->votes = take(pq ? BH * p->Cq * p->Ck * 4 : 0);
  L->pq_ws = take(pq ? ig::pq_scratch_bytes((int)BH, p->d, p->Ck) : 0);
  const size_t cq_ws = ig::kmeans_scratch_bytes(ig::kmeans_geom((int)BH, p->N, p->d, p->Cq));
  const size_t ck_ws = ig::kmeans_scratch_bytes(ig::kmeans_geom((int)BH, p->N, p->d, p->Ck));
  L->cluster_ws = take(cq_ws > ck_ws ? cq_ws : ck_ws);
  L->total = off;
  return IG_OK;
}

// bh0: global index of the first head (the sample's Philox counter uses it).
int select_impl(const float* cq, const float* ck, const int32_t* k_offsets, const instagen_params* p,
                int32_t* exact_groups, int32_t* counts, int32_t* sample_pos, float* sample_bias, int bh0,
                void* stream, const int32_t* votes = nullptr) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(p->Cq)) || (rc = check_clusters(p->Ck))) return rc;
  if ((rc = check_budgets(p))) return rc;
  const long long m = budget(p->sample_frac, p->N);
  if (!cq || !ck || !k_offsets || !exact_groups || !counts || !aligned16(ck)) return IG_ERR_INVALID_ARG;
  if (m > 0 && (!sample_pos || !sample_bias)) return IG_ERR_INVALID_ARG;
  ig::SelectArgs a;
  a.cq = cq;
  a.ck = ck;
  a.k_offsets = k_offsets;
  a.BH = p->B * p->H;
  a.Cq = p->Cq;
  a.Ck = p->Ck;
  a.d = p->d;
  a.scale = p->softmax_scale;
  a.E = budget(p->exact_frac, p->N);
  a.m = m;
  a.seed = p->seed;
  a.layer = p->layer;
  a.mode = p->sampling;
  a.bh0 = bh0;
  a.votes = votes;
  a.top_p = p->selection == IG_SELECT_TOP_P ? 1 : 0;
  a.p_fix = llround((double)p->top_p * 1048576.0);
  a.floor_keys = budget(p->key_floor, p->N);
  a.exact_groups = exact_groups;
  a.counts = counts;
  a.sample_pos = sample_pos;
  a.sample_bias = sample_bias;
  return cuda_status(ig::launch_select_sample(a, static_cast<cudaStream_t>(stream)));
}


// The whole call on device buffers; bh0 = global index of the first head;
// cq_init / ck_init: initial centroids or null (token floor(j*N/C)).
// k_ready / v_ready (may be null): events the stream waits for before the
// first kernel that reads K, and V, so that a caller copying Q, K and V in
// that order can start the query clustering once Q is in.
int forward_impl(const void* Q, const void* K, const void* V, void* O, const instagen_params* p,
                 const float* cq_init, const float* ck_init, void* ws, size_t ws_bytes, int bh0, void* stream,
                 cudaEvent_t k_ready = nullptr, cudaEvent_t v_ready = nullptr) {
  instagen_forward_layout L;
  int rc = forward_layout(p, &L);
  if (rc) return rc;
  if (p->Ck > ig::kAttnMaxExactGroups) return IG_ERR_UNSUPPORTED;
  if (p->kmeans_iters < 1 || p->kmeans_iters > 10000) return IG_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return IG_ERR_INVALID_ARG;
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return IG_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  float* cq = reinterpret_cast<float*>(w + L.cq);
  float* ck = reinterpret_cast<float*>(w + L.ck);
  int32_t* qa = reinterpret_cast<int32_t*>(w + L.q_assign);
  int32_t* ka = reinterpret_cast<int32_t*>(w + L.k_assign);
  int32_t* qp = reinterpret_cast<int32_t*>(w + L.q_perm);
  int32_t* kp = reinterpret_cast<int32_t*>(w + L.k_perm);
  int32_t* qo = reinterpret_cast<int32_t*>(w + L.q_offsets);
  int32_t* ko = reinterpret_cast<int32_t*>(w + L.k_offsets);
  void* Kp = w + L.kp;
  void* Vp = w + L.vp;
  int32_t* eg = reinterpret_cast<int32_t*>(w + L.exact_groups);
  int32_t* cnt = reinterpret_cast<int32_t*>(w + L.counts);
  int32_t* sp = reinterpret_cast<int32_t*>(w + L.sample_pos);
  float* sb = reinterpret_cast<float*>(w + L.sample_bias);
  void* cws = w + L.cluster_ws;
  const size_t cws_bytes = L.total - L.cluster_ws;
  rc = run_cluster(Q, p->Cq, p->kmeans_iters, cq_init, p, cq, qa, qp, qo, cws, cws_bytes, s);
  if (rc) return rc;
  if (k_ready && cudaStreamWaitEvent(s, k_ready, 0) != cudaSuccess) return IG_ERR_CUDA;
  rc = run_cluster(K, p->Ck, p->kmeans_iters, ck_init, p, ck, ka, kp, ko, cws, cws_bytes, s);
  if (rc) return rc;
  if (v_ready && cudaStreamWaitEvent(s, v_ready, 0) != cudaSuccess) return IG_ERR_CUDA;
  rc = cuda_status(ig::launch_gather_rows(static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V),
                                          kp, p->B * p->H, p->N, p->d, Kp, Vp, false, true, s));
  if (rc) return rc;
  int32_t* votes = nullptr;
  if (p->selection == IG_SELECT_PQ_VOTE) {
    votes = reinterpret_cast<int32_t*>(w + L.votes);
    rc = instagen_pq_votes(Q, cq, ck, qp, qo, ko, p, votes, w + L.pq_ws, L.cluster_ws - L.pq_ws, stream);
    if (rc) return rc;
  }
  rc = select_impl(cq, ck, ko, p, eg, cnt, sp, sb, bh0, stream, votes);
  if (rc) return rc;
  return instagen_attention(Q, Kp, Vp, qp, qo, ko, eg, cnt, sp, sb, p, O, stream);
}


// ------------------------------------------------------ host-buffer pipeline
// Staging slots of the host-buffer pipeline: chunk c uses slot c % 3, so the
// copy in of chunk c + 1 never waits for the compute of chunk c - 1.
constexpr int kHostSlots = 3;

struct HostLayout {
  int hc;                 // heads per chunk (at most)
  size_t tensor;          // bytes of one chunk of one tensor (256-aligned)
  size_t fwd_off, fwd;    // instagen_forward workspace of one chunk (one per slot)
  size_t total;
};

int host_layout(const instagen_params* p, int heads_per_chunk, HostLayout* L) {
  const size_t head_bytes = (size_t)p->N * p->d * 2;
  int hc = heads_per_chunk;
  if (hc <= 0) {  // about 160 MB per tensor per chunk
    const size_t k = ((size_t)160 << 20) / head_bytes;
    hc = (int)(k < 1 ? 1 : (k > (size_t)p->H ? (size_t)p->H : k));
  }
  if (hc > p->H) hc = p->H;
  instagen_params pc = *p;
  pc.B = 1;
  pc.H = hc;
  instagen_forward_layout fl;
  const int rc = forward_layout(&pc, &fl);
  if (rc) return rc;
  L->hc = hc;
  L->tensor = align256((size_t)hc * head_bytes);
  L->fwd_off = 4 * kHostSlots * L->tensor;  // slots x (Q, K, V, O)
  L->fwd = fl.total;
  L->total = L->fwd_off + kHostSlots * align256(fl.total);
  return IG_OK;
}

}  // namespace

extern "C" {

int64_t instagen_exact_budget(const instagen_params* p) {
  if (check_params(p)) return -1;
  return budget(p->exact_frac, p->N);
}

int64_t instagen_sample_budget(const instagen_params* p) {
  if (check_params(p)) return -1;
  return budget(p->sample_frac, p->N);
}

const char* instagen_error_string(int status) {
  switch (status) {
    case IG_OK: return "ok";
    case IG_ERR_INVALID_ARG: return "invalid argument";
    case IG_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case IG_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case IG_ERR_CUDA: return "CUDA runtime error";
    case IG_ERR_DEVICE_CHECK: return "device check failed (index out of range or wait timeout)";
    default: return "unknown status";
  }
}

int instagen_device_status(void* stream) {
  int v = 0;
  cudaError_t e = ig::read_and_clear_device_error(&v, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return IG_ERR_CUDA;
  return v ? IG_ERR_DEVICE_CHECK : IG_OK;
}

size_t instagen_cluster_workspace_size(const instagen_params* p, int32_t C) {
  if (check_params(p) || check_clusters(C)) return 0;
  return ig::kmeans_scratch_bytes(ig::kmeans_geom(p->B * p->H, p->N, p->d, C));
}

size_t instagen_workspace_size(const instagen_params* p) {
  instagen_forward_layout L;
  if (forward_layout(p, &L)) return 0;
  return L.total;
}

int instagen_forward_layout_get(const instagen_params* p, instagen_forward_layout* out) {
  if (!out) return IG_ERR_INVALID_ARG;
  return forward_layout(p, out);
}

int instagen_cluster(const void* X, int32_t C, int32_t iters, const float* init, const instagen_params* p,
                     float* centroids, int32_t* assign, int32_t* perm, int32_t* offsets, void* ws,
                     size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(C))) return rc;
  if (iters < 1 || iters > 10000) return IG_ERR_INVALID_ARG;
  if (!X || !centroids || !assign || !perm || !offsets || !aligned16(X)) return IG_ERR_INVALID_ARG;
  return run_cluster(X, C, iters, init, p, centroids, assign, perm, offsets, ws, ws_bytes,
                     static_cast<cudaStream_t>(stream));
}

int instagen_permutation(const int32_t* assign, int32_t C, const instagen_params* p, int32_t* perm,
                         int32_t* offsets, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(C))) return rc;
  if (!assign || !perm || !offsets) return IG_ERR_INVALID_ARG;
  return cuda_status(
      ig::launch_count_sort(assign, p->B * p->H, p->N, C, perm, offsets, nullptr, 0,
                            static_cast<cudaStream_t>(stream)));
}

int instagen_gather(const void* X, const int32_t* perm, const instagen_params* p, void* Xp, int32_t to_f16,
                    void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if (!X || !perm || !Xp || X == Xp || !aligned16(X) || !aligned16(Xp)) return IG_ERR_INVALID_ARG;
  if (to_f16 != 0 && to_f16 != 1) return IG_ERR_INVALID_ARG;
  return cuda_status(ig::launch_gather_rows(static_cast<const __nv_bfloat16*>(X), nullptr, perm, p->B * p->H,
                                            p->N, p->d, Xp, nullptr, to_f16 != 0, false,
                                            static_cast<cudaStream_t>(stream)));
}

size_t instagen_pq_votes_workspace_size(const instagen_params* p) {
  if (check_params(p) || check_clusters(p->Cq) || check_clusters(p->Ck)) return 0;
  return ig::pq_scratch_bytes(p->B * p->H, p->d, p->Ck);
}

int instagen_pq_votes(const void* Q, const float* cq, const float* ck, const int32_t* q_perm,
                      const int32_t* q_offsets, const int32_t* k_offsets, const instagen_params* p, int32_t* votes,
                      void* ws, size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(p->Cq)) || (rc = check_clusters(p->Ck))) return rc;
  if ((rc = check_budgets(p))) return rc;
  if (p->N > 0xFFFFF) return IG_ERR_UNSUPPORTED;
  if (!Q || !cq || !ck || !q_perm || !q_offsets || !k_offsets || !votes || !aligned16(Q)) return IG_ERR_INVALID_ARG;
  const int BH = p->B * p->H;
  if (!ws || ws_bytes < ig::pq_scratch_bytes(BH, p->d, p->Ck) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return IG_ERR_WORKSPACE;
  ig::PqArgs a;
  a.cq = cq;
  a.ck = ck;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.q_perm = q_perm;
  a.q_offsets = q_offsets;
  a.k_offsets = k_offsets;
  a.BH = BH;
  a.N = p->N;
  a.d = p->d;
  a.Cq = p->Cq;
  a.Ck = p->Ck;
  a.E = budget(p->exact_frac, p->N);
  a.codebooks = nullptr;
  a.kcodes = nullptr;
  a.votes = votes;
  return cuda_status(ig::launch_pq_votes(a, ws, static_cast<cudaStream_t>(stream)));
}

int instagen_select_sample_votes(const float* cq, const float* ck, const int32_t* k_offsets, const int32_t* votes,
                                 const instagen_params* p, int32_t* exact_groups, int32_t* counts,
                                 int32_t* sample_pos, float* sample_bias, void* stream) {
  if (!votes) return IG_ERR_INVALID_ARG;
  return select_impl(cq, ck, k_offsets, p, exact_groups, counts, sample_pos, sample_bias, 0, stream, votes);
}

int instagen_select_sample(const float* cq, const float* ck, const int32_t* k_offsets, const instagen_params* p,
                           int32_t* exact_groups, int32_t* counts, int32_t* sample_pos, float* sample_bias,
                           void* stream) {
  return select_impl(cq, ck, k_offsets, p, exact_groups, counts, sample_pos, sample_bias, 0, stream);
}

int instagen_attention(const void* Q, const void* Kp, const void* Vp, const int32_t* q_perm,
                       const int32_t* q_offsets, const int32_t* k_offsets, const int32_t* exact_groups,
                       const int32_t* counts, const int32_t* sample_pos, const float* sample_bias,
                       const instagen_params* p, void* O, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(p->Cq)) || (rc = check_clusters(p->Ck))) return rc;
  if (p->Ck > ig::kAttnMaxExactGroups) return IG_ERR_UNSUPPORTED;
  if ((rc = check_budgets(p))) return rc;
  const long long m = budget(p->sample_frac, p->N);
  if (!Q || !Kp || !Vp || !q_perm || !q_offsets || !k_offsets || !exact_groups || !counts || !O)
    return IG_ERR_INVALID_ARG;
  if (m > 0 && (!sample_pos || !sample_bias)) return IG_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kp) || !aligned16(Vp) || !aligned16(O)) return IG_ERR_INVALID_ARG;
  ig::AttnArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.Kp = static_cast<const __nv_bfloat16*>(Kp);
  a.Vp = static_cast<const __half*>(Vp);
  a.q_perm = q_perm;
  a.q_offsets = q_offsets;
  a.k_offsets = k_offsets;
  a.exact_groups = exact_groups;
  a.counts = counts;
  a.sample_pos = sample_pos;
  a.sample_bias = sample_bias;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.BH = p->B * p->H;
  a.N = p->N;
  a.d = p->d;
  a.Cq = p->Cq;
  a.Ck = p->Ck;
  a.m = m;
  a.scale_log2 = p->softmax_scale * 1.4426950408889634f;
  return cuda_status(ig::launch_attention(a, static_cast<cudaStream_t>(stream)));
}

int instagen_forward(const void* Q, const void* K, const void* V, void* O, const instagen_params* p, void* ws,
                     size_t ws_bytes, void* stream) {
  return forward_impl(Q, K, V, O, p, nullptr, nullptr, ws, ws_bytes, 0, stream);
}

int instagen_forward_init(const void* Q, const void* K, const void* V, void* O, const instagen_params* p,
                          const float* cq_init, const float* ck_init, void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(Q, K, V, O, p, cq_init, ck_init, ws, ws_bytes, 0, stream);
}

size_t instagen_forward_host_workspace_size(const instagen_params* p, int32_t heads_per_chunk) {
  HostLayout L;
  if (check_params(p) || heads_per_chunk < 0 || host_layout(p, heads_per_chunk, &L)) return 0;
  return L.total;
}

int instagen_forward_host(const void* Q, const void* K, const void* V, void* O, const instagen_params* p,
                          int32_t heads_per_chunk, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if (heads_per_chunk < 0 || !Q || !K || !V || !O) return IG_ERR_INVALID_ARG;
  HostLayout L;
  if ((rc = host_layout(p, heads_per_chunk, &L))) return rc;
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return IG_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr, s_c1 = nullptr;
  // start, Q in[], K in[], V in[], comp[], out[], in done, out done, compute-1 done
  constexpr int kEv = 4 + 5 * kHostSlots;
  cudaEvent_t ev[kEv] = {};
  bool ok = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&s_c1, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; i < kEv && ok; ++i) ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
  cudaEvent_t ev_start = ev[0], *ev_in = ev + 1, *ev_in_k = ev + 1 + kHostSlots, *ev_in_v = ev + 1 + 2 * kHostSlots;
  cudaEvent_t *ev_comp = ev + 1 + 3 * kHostSlots, *ev_out = ev + 1 + 4 * kHostSlots;
  cudaEvent_t ev_in_done = ev[kEv - 3], ev_out_done = ev[kEv - 2], ev_c1_done = ev[kEv - 1];
  // chunks alternate between two compute streams (the caller's and one of
  // ours), each with its own forward workspace, so one chunk's tail overlaps
  // the next chunk's first kernels
  rc = ok ? IG_OK : IG_ERR_CUDA;
  char* w = static_cast<char*>(ws);
  const size_t head_bytes = (size_t)p->N * p->d * 2;
  const char* hq = static_cast<const char*>(Q);
  const char* hk = static_cast<const char*>(K);
  const char* hv = static_cast<const char*>(V);
  char* ho = static_cast<char*>(O);
  if (rc == IG_OK) {
    ok = cudaEventRecord(ev_start, s) == cudaSuccess && cudaStreamWaitEvent(s_in, ev_start, 0) == cudaSuccess &&
         cudaStreamWaitEvent(s_out, ev_start, 0) == cudaSuccess &&
         cudaStreamWaitEvent(s_c1, ev_start, 0) == cudaSuccess;
    if (!ok) rc = IG_ERR_CUDA;
  }
  // chunk sizes of a batch row: one head first, so the GPU starts after one
  // head's copy in; then each chunk half again as large as the one before, up
  // to hc, so that (the copy in of a head being faster than its compute) the
  // next chunk is in before this one is computed; and one head last, a short
  // drain.  Small chunks cost a little (smaller grids, more launches), the
  // growth keeps their number logarithmic in hc.
  auto chunk_at = [&](int h, int prev) {
    const int left = p->H - h;
    if (h == 0 || left <= 1) return 1;
    int n = (3 * prev + 1) / 2;
    if (n < prev + 1) n = prev + 1;
    if (n > L.hc) n = L.hc;
    return left <= n + 1 ? left - 1 : n;
  };
  int c = 0;
  for (int b = 0; b < p->B && rc == IG_OK; ++b) {
    for (int h0 = 0, n = 0; h0 < p->H && rc == IG_OK; h0 += n, ++c) {
      n = chunk_at(h0, n);
      const int slot = c % kHostSlots;
      const size_t off = ((size_t)b * p->H + h0) * head_bytes, bytes = (size_t)n * head_bytes;
      char* dq = w + (4 * slot + 0) * L.tensor;
      char* dk = w + (4 * slot + 1) * L.tensor;
      char* dv = w + (4 * slot + 2) * L.tensor;
      char* dout = w + (4 * slot + 3) * L.tensor;
      // copy in: the slot's inputs are free once chunk c - kHostSlots is computed
      // (an event after each tensor: the chunk's query clustering starts once
      // Q is in, while K and V are still being copied)
      ok = (c < kHostSlots || cudaStreamWaitEvent(s_in, ev_comp[slot], 0) == cudaSuccess) &&
           cudaMemcpyAsync(dq, hq + off, bytes, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
           cudaEventRecord(ev_in[slot], s_in) == cudaSuccess &&
           cudaMemcpyAsync(dk, hk + off, bytes, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
           cudaEventRecord(ev_in_k[slot], s_in) == cudaSuccess &&
           cudaMemcpyAsync(dv, hv + off, bytes, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
           cudaEventRecord(ev_in_v[slot], s_in) == cudaSuccess;
      // compute (consecutive chunks alternate between two streams): after
      // Q's copy in (K's and V's are waited for inside), and once chunk
      // c - kHostSlots's output left the slot
      cudaStream_t cs = (c & 1) ? s_c1 : s;
      ok = ok && cudaStreamWaitEvent(cs, ev_in[slot], 0) == cudaSuccess &&
           (c < kHostSlots || cudaStreamWaitEvent(cs, ev_out[slot], 0) == cudaSuccess);
      if (!ok) {
        rc = IG_ERR_CUDA;
        break;
      }
      instagen_params pc = *p;
      pc.B = 1;
      pc.H = n;
      rc = forward_impl(dq, dk, dv, dout, &pc, nullptr, nullptr, w + L.fwd_off + slot * align256(L.fwd), L.fwd,
                        b * p->H + h0, cs, ev_in_k[slot], ev_in_v[slot]);
      if (rc) break;
      // copy out
      ok = cudaEventRecord(ev_comp[slot], cs) == cudaSuccess &&
           cudaStreamWaitEvent(s_out, ev_comp[slot], 0) == cudaSuccess &&
           cudaMemcpyAsync(ho + off, dout, bytes, cudaMemcpyDeviceToHost, s_out) == cudaSuccess &&
           cudaEventRecord(ev_out[slot], s_out) == cudaSuccess;
      if (!ok) rc = IG_ERR_CUDA;
    }
  }
  // `stream` is ordered after everything enqueued on the copy streams, also
  // on an error (so synchronising it covers every pending host access)
  if (s_in && ev_in_done && cudaEventRecord(ev_in_done, s_in) == cudaSuccess) cudaStreamWaitEvent(s, ev_in_done, 0);
  if (s_out && ev_out_done && cudaEventRecord(ev_out_done, s_out) == cudaSuccess)
    cudaStreamWaitEvent(s, ev_out_done, 0);
  if (s_c1 && ev_c1_done && cudaEventRecord(ev_c1_done, s_c1) == cudaSuccess) cudaStreamWaitEvent(s, ev_c1_done, 0);
  for (int i = 0; i < kEv; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);  // released once their work completes
  if (s_in) cudaStreamDestroy(s_in);
  if (s_out) cudaStreamDestroy(s_out);
  if (s_c1) cudaStreamDestroy(s_c1);
  return rc;
}
}  // extern "C"
