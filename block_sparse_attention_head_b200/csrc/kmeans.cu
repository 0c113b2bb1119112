// Batched k-means for the query / key clustering of InstaGen (thelatestinai.com
// paper page, Figure 3 (a): "queries and keys are clustered into groups";
// Figure 2 caption: Cq = 100, Ck = 500).
//
// One Lloyd iteration = assign (tensor cores) -> stable counting sort ->
// deterministic per-cluster mean.  Distances: ||x - c||^2 = ||x||^2 + ||c||^2
// - 2 x.c; ||x||^2 is common to a token's candidates, so the argmin runs over
// ||c||^2 - 2 x.c.  x.c is one tcgen05 GEMM with K = 2d: the bf16 token row is
// multiplied by the centroid split into bf16 hi and lo halves (hi + lo carries
// ~16 mantissa bits of the fp32 centroid), accumulated in fp32 in TMEM.
#include "internal.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace ig {

KmeansGeom kmeans_geom(int BH, int N, int d, int C) {
  KmeansGeom g;
  g.BH = BH;
  g.N = N;
  g.d = d;
  g.C = C;
  int c16 = (C + 15) / 16 * 16;
  g.chunk = c16 < 128 ? c16 : 128;
  g.c_pad = (C + g.chunk - 1) / g.chunk * g.chunk;
  return g;
}

// Rows summed by one CTA of the update; clusters with more members are split
// into pieces of this many rows (in permuted order) whose partial sums are
// added in piece order.
constexpr int kUpdRows = 2048;

// Partial-sum slots per head: the pieces of every cluster larger than one
// piece.  A cluster of n > R rows has ceil(n/R) < 2n/R pieces, so all of them
// together stay below 2N/R.
int kmeans_part_slots(const KmeansGeom& g) { return (int)((2LL * g.N) / kUpdRows + 1); }

namespace {
size_t a256(size_t b) { return (b + 255) / 256 * 256; }
}  // namespace

size_t kmeans_scratch_bytes(const KmeansGeom& g) {
  const size_t BH = (size_t)g.BH;
  return a256(BH * g.c_pad * 2 * g.d * sizeof(__nv_bfloat16)) + a256(BH * g.c_pad * sizeof(float)) +
         a256(BH * kmeans_part_slots(g) * g.d * sizeof(float)) + a256(BH * g.C * sizeof(int32_t));
}

KmeansScratch kmeans_scratch_carve(const KmeansGeom& g, void* ws) {
  const size_t BH = (size_t)g.BH;
  char* b = static_cast<char*>(ws);
  KmeansScratch sc;
  sc.cmma = reinterpret_cast<__nv_bfloat16*>(b);
  b += a256(BH * g.c_pad * 2 * g.d * sizeof(__nv_bfloat16));
  sc.norms = reinterpret_cast<float*>(b);
  b += a256(BH * g.c_pad * sizeof(float));
  sc.partial = reinterpret_cast<float*>(b);
  b += a256(BH * kmeans_part_slots(g) * g.d * sizeof(float));
  sc.arrive = reinterpret_cast<int32_t*>(b);
  return sc;
}

// Writes the hi/lo bf16 operand row and ||c||^2 for centroid row `c` (one warp).
__device__ __forceinline__ void write_operand_row(const float* c, int d, __nv_bfloat16* hi_lo, float* norm,
                                                  int lane) {
  float ss = 0.f;
  for (int k = lane; k < d; k += 32) {
    float v = c[k];
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    hi_lo[k] = h;
    hi_lo[d + k] = l;
    ss = fmaf(v, v, ss);
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) *norm = ss;
}

// Initial centroids (given, or token floor(j*N/C)) and their operand rows.
// One warp per (bh, padded centroid row).
__global__ void kmeans_init_kernel(KmeansGeom g, const __nv_bfloat16* __restrict__ X, const float* __restrict__ init,
                                   float* __restrict__ cent, __nv_bfloat16* __restrict__ cmma,
                                   float* __restrict__ norms, int32_t* __restrict__ arrive) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int total = g.BH * g.c_pad;
  if (warp >= total) return;
  const int bh = warp / g.c_pad, j = warp % g.c_pad;
  if (j < g.C && lane == 0) arrive[(size_t)bh * g.C + j] = 0;
  __nv_bfloat16* op = cmma + ((size_t)bh * g.c_pad + j) * 2 * g.d;
  if (j >= g.C) {  // padding row: zero operand, never selected
    for (int k = lane; k < 2 * g.d; k += 32) op[k] = __float2bfloat16_rn(0.f);
    if (lane == 0) norms[(size_t)bh * g.c_pad + j] = 0.f;
    return;
  }
  float* c = cent + ((size_t)bh * g.C + j) * g.d;
  if (init) {
    const float* src = init + ((size_t)bh * g.C + j) * g.d;
    for (int k = lane; k < g.d; k += 32) c[k] = src[k];
  } else {
    const long long tok = ((long long)j * g.N) / g.C;
    const __nv_bfloat16* src = X + ((size_t)bh * g.N + tok) * g.d;
    for (int k = lane; k < g.d; k += 32) c[k] = __bfloat162float(src[k]);
  }
  __syncwarp();
  write_operand_row(c, g.d, op, norms + (size_t)bh * g.c_pad + j, lane);
}

cudaError_t launch_kmeans_init(const KmeansGeom& g, const __nv_bfloat16* X, const float* init, float* cent,
                               const KmeansScratch& sc, cudaStream_t s) {
  const long long warps = (long long)g.BH * g.c_pad;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  kmeans_init_kernel<<<(unsigned)blocks, threads, 0, s>>>(g, X, init, cent, sc.cmma, sc.norms, sc.arrive);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ assign
// CTA = up to kPairsPerCta pairs of 128-token tiles of one head (M = 2 x 128),
// streaming the head's centroid operand through shared memory in K-blocks of
// 64 columns (TMA, 128-byte swizzle) for each chunk of <= 128 centroids.
// TMEM: 2 buffers x 2 tiles x 128 fp32 columns; the epilogue of chunk c
// (argmin over the chunk's columns) overlaps the MMAs of chunk c+1.
// Warps: 0 TMA producer, 1 MMA issuer (+ TMEM owner), 4-7 epilogue tile 0,
// 8-11 epilogue tile 1; warps 2-3 only join the block-wide barriers.
namespace {
constexpr int kAssignThreads = 384;
constexpr int kAssignStages = 4;
constexpr int kPairsPerCta = 4;

template <int D>
struct AssignSmem {
  static constexpr int kXBlocks = D / 64;                 // 64-column K-blocks of a token tile
  static constexpr int kXTileBytes = kXBlocks * 128 * 128;  // 128 rows x D bf16
  static constexpr int kStageBytes = 128 * 128;           // <= 128 centroid rows x 64 columns
  static constexpr int kX = 0;
  static constexpr int kStages = kX + 2 * kXTileBytes;
  static constexpr int kBars = kStages + kAssignStages * kStageBytes;
  static constexpr int kNumBars = 2 * kAssignStages + 2 + 2 + 2 + 1;  // c_full, c_empty, x_full, x_empty, t_full, t_empty, fin
  static constexpr int kMisc = kBars + kNumBars * 8;            // tmem base, abort flag
  static constexpr int kNorms = kMisc + 16;
  static size_t bytes(int c_pad) { return 1024 + kNorms + (size_t)c_pad * 4; }
};
}  // namespace

template <int D>
__global__ void __launch_bounds__(kAssignThreads, 1)
    kmeans_assign_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                         KmeansGeom g, const float* __restrict__ norms, int32_t* __restrict__ assign) {
  using L = AssignSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* c_full = bars;
  uint64_t* c_empty = bars + kAssignStages;
  uint64_t* x_full = bars + 2 * kAssignStages;
  uint64_t* x_empty = x_full + 1;
  uint64_t* t_full = x_full + 2;   // [2] per TMEM buffer
  uint64_t* t_empty = x_full + 4;  // [2]
  uint64_t* fin = x_full + 6;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  float* norm_s = reinterpret_cast<float*>(smem + L::kNorms);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int pairs_total = (g.N + 255) / 256;
  const int pair0 = blockIdx.x * kPairsPerCta;
  const int npairs = min(kPairsPerCta, pairs_total - pair0);
  if (npairs <= 0) return;
  const int nchunks = g.c_pad / g.chunk;
  const int kblocks = 2 * L::kXBlocks;  // hi blocks then lo blocks

  for (int j = tid; j < g.c_pad; j += blockDim.x) norm_s[j] = norms[(size_t)bh * g.c_pad + j];
  if (tid == 0) {
    for (int s = 0; s < kAssignStages; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 1);
    }
    mbar_init(x_full, 1);
    mbar_init(x_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], 256);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t x_base = smem_u32(smem + L::kX);
  const uint32_t st_base = smem_u32(smem + L::kStages);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_c);
    int st = 0;
    bool ok = true;
    for (int pp = 0; pp < npairs && ok; ++pp) {
      if (pp > 0 && !mbar_wait(x_empty, (pp - 1) & 1, abort_flag)) break;
      const int row0 = bh * g.N + (pair0 + pp) * 256;
      mbar_arrive_expect_tx(x_full, 2 * L::kXTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int kb = 0; kb < L::kXBlocks; ++kb)
          tma_load_2d(x_base + t * L::kXTileBytes + kb * 16384, &tmap_x, kb * 64, row0 + t * 128, x_full);
      for (int c = 0; c < nchunks && ok; ++c) {
        for (int kb = 0; kb < kblocks; ++kb, ++st) {
          const int s = st % kAssignStages;
          if (st >= kAssignStages && !mbar_wait(&c_empty[s], ((st / kAssignStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&c_full[s], g.chunk * 128);
          tma_load_2d(st_base + s * L::kStageBytes, &tmap_c, kb * 64, bh * g.c_pad + c * g.chunk, &c_full[s]);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // -------------------------------------------------------------- MMA
    const uint32_t idesc = umma_idesc_bf16(128, g.chunk, false, false);
    int st = 0, gc = 0;  // stage counter, global chunk counter (TMEM buffer phases)
    bool ok = true;
    for (int pp = 0; pp < npairs && ok; ++pp) {
      if (!mbar_wait(x_full, pp & 1, abort_flag)) break;
      for (int c = 0; c < nchunks && ok; ++c, ++gc) {
        const int b = gc & 1;
        if (gc >= 2 && !mbar_wait(&t_empty[b], ((gc >> 1) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb, ++st) {
          const int s = st % kAssignStages;
          if (!mbar_wait(&c_full[s], (st / kAssignStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int xkb = kb % L::kXBlocks;
          for (int t = 0; t < 2; ++t) {
            const uint32_t dcol = tmem + (uint32_t)((b * 2 + t) * 128);
            for (int k = 0; k < 4; ++k) {
              const uint64_t adesc =
                  umma_desc_sw128(x_base + t * L::kXTileBytes + xkb * 16384 + k * 32, 16, 1024);
              const uint64_t bdesc = umma_desc_sw128(st_base + s * L::kStageBytes + k * 32, 16, 1024);
              umma_bf16_ss(dcol, adesc, bdesc, idesc, (kb | k) != 0);
            }
          }
          umma_commit(&c_empty[s]);
        }
        if (!ok) break;
        umma_commit(&t_full[b]);
      }
      if (ok) umma_commit(x_empty);
    }
    // drain: every issued MMA completes before TMEM is released
    umma_commit(fin);
    mbar_wait_drain(fin, 0);
  } else if (warp >= 4) {
    // --------------------------------------------------------- epilogue
    const int t = (warp - 4) >> 2;          // tile 0 or 1
    const int r = tid - 128 - t * 128;      // row inside the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((r & ~31) << 16);
    int gc = 0;
    bool ok = true;
    for (int pp = 0; pp < npairs && ok; ++pp) {
      float best = __int_as_float(0x7f800000);
      int best_j = 0;
      for (int c = 0; c < nchunks; ++c, ++gc) {
        const int b = gc & 1;
        if (!mbar_wait_warp(&t_full[b], (gc >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col0 = tmem + lane_off + (uint32_t)((b * 2 + t) * 128);
        for (int cb = 0; cb < g.chunk; cb += 32) {
          float v[32];
          tmem_ld32(col0 + cb, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = c * g.chunk + cb + e;
            if (cb + e < g.chunk && j < g.C) {
              const float dist = fmaf(-2.f, v[e], norm_s[j]);
              if (dist < best) {
                best = dist;
                best_j = j;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&t_empty[b]);
      }
      if (!ok) break;
      const int tok = (pair0 + pp) * 256 + t * 128 + r;
      if (tok < g.N) assign[(size_t)bh * g.N + tok] = best_j;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_kmeans_assign(const KmeansGeom& g, const CUtensorMap* tmap_x, const CUtensorMap* tmap_c,
                                 const float* norms, int32_t* assign, cudaStream_t s) {
  const int pairs = (g.N + 255) / 256;
  dim3 grid((pairs + kPairsPerCta - 1) / kPairsPerCta, g.BH);
  if (g.d == 128) {
    const size_t sm = AssignSmem<128>::bytes(g.c_pad);
    cudaError_t e = cudaFuncSetAttribute(kmeans_assign_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
    if (e != cudaSuccess) return e;
    kmeans_assign_kernel<128><<<grid, kAssignThreads, sm, s>>>(*tmap_x, *tmap_c, g, norms, assign);
  } else {
    const size_t sm = AssignSmem<64>::bytes(g.c_pad);
    cudaError_t e = cudaFuncSetAttribute(kmeans_assign_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
    if (e != cudaSuccess) return e;
    kmeans_assign_kernel<64><<<grid, kAssignThreads, sm, s>>>(*tmap_x, *tmap_c, g, norms, assign);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ update
// A grid over row pieces: a cluster of n members gets ceil(n/R) pieces of at
// most R = kUpdRows consecutive permuted rows (an empty cluster one empty
// piece), so the work of a CTA stays bounded however skewed the cluster sizes
// are.  A CTA finds its (cluster, piece) by a scan over the cluster sizes and
// sums its rows in kUpdThreads / (d/8) row slots, each slot a fixed
// subsequence of rows, the slot sums added in slot order.  A single-piece
// cluster writes its mean at once (an empty one keeps its centroid); the
// pieces of a larger cluster store their sums, and the CTA that arrives last
// adds them in piece order and writes the mean.  Every sum runs in a fixed
// order, so the centroids do not depend on scheduling.
constexpr int kUpdThreads = 256;
constexpr int kUpdUnroll = 4;  // rows in flight per slot

__device__ __forceinline__ int update_pieces(int n) { return n <= kUpdRows ? 1 : (n + kUpdRows - 1) / kUpdRows; }

__global__ void __launch_bounds__(kUpdThreads)
    kmeans_update_kernel(KmeansGeom g, const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm,
                         const int32_t* __restrict__ offsets, float* __restrict__ cent,
                         __nv_bfloat16* __restrict__ cmma, float* __restrict__ norms, float* __restrict__ partial,
                         int32_t* __restrict__ arrive, int part_slots) {
  __shared__ float part[kUpdThreads * 8];
  __shared__ float red[32];
  __shared__ int scan_np[kUpdThreads / 32], scan_mp[kUpdThreads / 32];
  __shared__ int s_c, s_piece, s_np, s_base, s_last;
  const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int32_t* off = offsets + (size_t)bh * (g.C + 1);

  // (cluster, piece) of this CTA: exclusive scans over the clusters of the
  // piece count and of the pieces that belong to multi-piece clusters
  const int per = (g.C + kUpdThreads - 1) / kUpdThreads;
  const int c0 = min(tid * per, g.C), c1 = min(c0 + per, g.C);
  int np_own = 0, mp_own = 0;
  for (int c = c0; c < c1; ++c) {
    const int k = update_pieces(max(off[c + 1] - off[c], 0));
    np_own += k;
    if (k > 1) mp_own += k;
  }
  int np_inc = np_own, mp_inc = mp_own;
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, np_inc, o);
    const int b = __shfl_up_sync(0xffffffffu, mp_inc, o);
    if (lane >= o) {
      np_inc += a;
      mp_inc += b;
    }
  }
  if (lane == 31) {
    scan_np[wid] = np_inc;
    scan_mp[wid] = mp_inc;
  }
  if (tid == 0) s_c = -1;
  __syncthreads();
  int at = np_inc - np_own, mb = mp_inc - mp_own;
  for (int w = 0; w < wid; ++w) {
    at += scan_np[w];
    mb += scan_mp[w];
  }
  const int t = blockIdx.x;
  if (t >= at && t < at + np_own) {
    for (int c = c0; c < c1; ++c) {
      const int k = update_pieces(max(off[c + 1] - off[c], 0));
      if (t < at + k) {
        s_c = c;
        s_piece = t - at;
        s_np = k;
        s_base = mb;
        break;
      }
      at += k;
      if (k > 1) mb += k;
    }
  }
  __syncthreads();
  const int c = s_c;
  if (c < 0) return;  // past the last piece of this head
  const int piece = s_piece, npieces = s_np;
  if (npieces > 1 && s_base + npieces > part_slots) {  // offsets that do not sum to N
    if (tid == 0) raise_error(kErrIndex);
    return;
  }

  const int cpr = g.d / 8;  // 16-byte chunks per row
  const int slots = kUpdThreads / cpr;
  const int slot = tid / cpr, ch = tid % cpr;
  const int lo = off[c], hi = off[c + 1];
  const int plo = lo + piece * kUpdRows, phi = min(hi, plo + kUpdRows);
  const int32_t* prow = perm + (size_t)bh * g.N;
  const __nv_bfloat16* xh = X + (size_t)bh * g.N * g.d + ch * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int p0 = plo + slot; p0 < phi; p0 += kUpdUnroll * slots) {
    int src[kUpdUnroll];
    uint4 raw[kUpdUnroll];
#pragma unroll
    for (int u = 0; u < kUpdUnroll; ++u) {
      const int p = p0 + u * slots;
      src[u] = p < phi ? prow[p] : -1;
    }
#pragma unroll
    for (int u = 0; u < kUpdUnroll; ++u) {
      const bool live = p0 + u * slots < phi;
      const bool ok = src[u] >= 0 && src[u] < g.N;
      if (live && !ok) raise_error(kErrIndex);
      raw[u] = (live && ok) ? *reinterpret_cast<const uint4*>(xh + (size_t)src[u] * g.d) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUpdUnroll; ++u) {  // rows added in permuted order
      if (p0 + u * slots >= phi) break;
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[slot * g.d + ch * 8 + e] = acc[e];
  __syncthreads();
  float sum = 0.f;
  if (tid < g.d)
    for (int sl = 0; sl < slots; ++sl) sum += part[sl * g.d + tid];

  if (npieces > 1) {
    float* pbase = partial + ((size_t)bh * part_slots + s_base) * g.d;
    if (tid < g.d) pbase[(size_t)piece * g.d + tid] = sum;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&arrive[(size_t)bh * g.C + c], 1) == npieces - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid < g.d) {
      sum = 0.f;
      for (int q = 0; q < npieces; ++q) sum += __ldcg(pbase + (size_t)q * g.d + tid);
    }
    if (tid == 0) arrive[(size_t)bh * g.C + c] = 0;  // ready for the next update
  }

  const int n = hi - lo;
  float sq = 0.f;
  if (tid < g.d) {
    float* cr = cent + ((size_t)bh * g.C + c) * g.d;
    float v;
    if (n > 0) {
      v = sum / (float)n;
      cr[tid] = v;
    } else {
      v = cr[tid];  // empty cluster keeps its centroid
    }
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    __nv_bfloat16* op = cmma + ((size_t)bh * g.c_pad + c) * 2 * g.d;
    op[tid] = h;
    op[g.d + tid] = l;
    sq = v * v;
  }
  // ||c||^2: warp sums then a fixed-order sum of the warp partials
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0) red[wid] = sq;
  __syncthreads();
  if (tid == 0) {
    float tot = 0.f;
    for (int w = 0; w < (g.d + 31) / 32; ++w) tot += red[w];
    norms[(size_t)bh * g.c_pad + c] = tot;
  }
}

cudaError_t launch_kmeans_update(const KmeansGeom& g, const __nv_bfloat16* X, const int32_t* perm,
                                 const int32_t* offsets, float* cent, const KmeansScratch& sc, cudaStream_t s) {
  // at most C + N/R pieces per head (every cluster adds at most one piece
  // beyond n/R); CTAs past a head's last piece return at once
  dim3 grid(g.C + (g.N + kUpdRows - 1) / kUpdRows, g.BH);
  kmeans_update_kernel<<<grid, kUpdThreads, 0, s>>>(g, X, perm, offsets, cent, sc.cmma, sc.norms, sc.partial,
                                                     sc.arrive, kmeans_part_slots(g));
  return cudaGetLastError();
}

}  // namespace ig
