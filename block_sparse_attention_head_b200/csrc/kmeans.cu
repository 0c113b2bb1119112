// Batched k-means for the query / key clustering of InstaGen (thelatestinai.com
// paper page, Figure 3 (a): both the queries and the keys are partitioned by
// clustering; Figure 2 caption: Cq = 100, Ck = 500).
//
// One Lloyd iteration = assign (tensor cores) -> stable counting sort ->
// deterministic per-cluster mean.  Distances: ||x - c||^2 = ||x||^2 + ||c||^2
// - 2 x.c; ||x||^2 is common to a token's candidates, so the argmin runs over
// ||c||^2 - 2 x.c, i.e. the argmax of x.c - ||c||^2 / 2.  x.c is one tcgen05
// GEMM with K = 2d: the bf16 token row is multiplied by the centroid split
// into bf16 hi and lo halves (hi + lo carries ~16 mantissa bits of the fp32
// centroid), accumulated in fp32 in TMEM, and one more K = 16 step adds
// -||c||^2 / 2 from the centroid's norm row.
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
  // chunks of <= 256 centroids (one MMA's N), as few and as even as possible,
  // each a multiple of 16 so that each CTA of a pair holds whole 8-row groups
  const int c16 = (C + 15) / 16 * 16;
  const int nch = (c16 + 255) / 256;
  g.chunk = ((c16 + nch - 1) / nch + 15) / 16 * 16;
  g.c_pad = nch * g.chunk;
  return g;
}


// Partial-sum slots per head: the pieces of every cluster larger than one
// piece.  A cluster of n > R rows has ceil(n/R) < 2n/R pieces, so all of them
// together stay below 2N/R.
int kmeans_part_slots(const KmeansGeom& g) { return (int)((2LL * g.N) / kUpdRows + 1); }

namespace {
size_t a256(size_t b) { return (b + 255) / 256 * 256; }
}  // namespace

size_t kmeans_scratch_bytes(const KmeansGeom& g) {
  const size_t BH = (size_t)g.BH;
  return a256(BH * g.c_pad * 2 * g.d * sizeof(__nv_bfloat16)) + a256(BH * g.c_pad * kNormCols * sizeof(__nv_bfloat16)) +
         a256(BH * kmeans_update_grid(g) * sizeof(int4)) +
         a256(BH * kmeans_part_slots(g) * g.d * sizeof(float)) + a256(BH * g.C * sizeof(int32_t));
}

KmeansScratch kmeans_scratch_carve(const KmeansGeom& g, void* ws) {
  const size_t BH = (size_t)g.BH;
  char* b = static_cast<char*>(ws);
  KmeansScratch sc;
  sc.cmma = reinterpret_cast<__nv_bfloat16*>(b);
  b += a256(BH * g.c_pad * 2 * g.d * sizeof(__nv_bfloat16));
  sc.nrow = reinterpret_cast<__nv_bfloat16*>(b);
  b += a256(BH * g.c_pad * kNormCols * sizeof(__nv_bfloat16));
  sc.pmap = reinterpret_cast<int4*>(b);
  b += a256(BH * kmeans_update_grid(g) * sizeof(int4));
  sc.partial = reinterpret_cast<float*>(b);
  b += a256(BH * kmeans_part_slots(g) * g.d * sizeof(float));
  sc.arrive = reinterpret_cast<int32_t*>(b);
  return sc;
}

// Lane `lane` (0-31) of a warp writes column `lane` of a centroid's norm row
// for ||c||^2 = ss (every lane holds ss); an infinite ss makes a padding row.
__device__ __forceinline__ void write_norm_row(float ss, __nv_bfloat16* nrow, int lane) {
  const int k = lane & 15;
  float t = 0.f;
  if (lane < 16 && (k == 0 || k == 8) && isinf(ss)) {
    t = -ss;
  } else if (lane < 16 && isfinite(ss) && (k & 7) < 3) {
    // -ss / 4 = t0 + t1 + t2, each rounded to bf16 in turn
    const float v = -0.25f * ss;
    const float t0 = __bfloat162float(__float2bfloat16_rn(v));
    const float t1 = __bfloat162float(__float2bfloat16_rn(v - t0));
    const float t2 = __bfloat162float(__float2bfloat16_rn((v - t0) - t1));
    t = (k & 7) == 0 ? t0 : (k & 7) == 1 ? t1 : t2;
  }
  nrow[lane] = __float2bfloat16_rn(t);
}

// Writes the hi/lo bf16 operand row and the norm row for centroid row `c`
// (one warp).
__device__ __forceinline__ void write_operand_row(const float* c, int d, __nv_bfloat16* hi_lo, __nv_bfloat16* nrow,
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
  write_norm_row(ss, nrow, lane);
}

// Initial centroids (given, or token floor(j*N/C)) and their operand rows.
// One warp per (bh, padded centroid row).
__global__ void kmeans_init_kernel(KmeansGeom g, const __nv_bfloat16* __restrict__ X, const float* __restrict__ init,
                                   float* __restrict__ cent, __nv_bfloat16* __restrict__ cmma,
                                   __nv_bfloat16* __restrict__ nrows, int32_t* __restrict__ arrive) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int total = g.BH * g.c_pad;
  if (warp >= total) return;
  const int bh = warp / g.c_pad, j = warp % g.c_pad;
  if (j < g.C && lane == 0) arrive[(size_t)bh * g.C + j] = 0;
  __nv_bfloat16* op = cmma + ((size_t)bh * g.c_pad + j) * 2 * g.d;
  __nv_bfloat16* nr = nrows + ((size_t)bh * g.c_pad + j) * kNormCols;
  if (j >= g.C) {  // padding row: zero operand, infinite norm, never selected
    for (int k = lane; k < 2 * g.d; k += 32) op[k] = __float2bfloat16_rn(0.f);
    write_norm_row(__int_as_float(0x7f800000), nr, lane);
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
  write_operand_row(c, g.d, op, nr, lane);
}

cudaError_t launch_kmeans_init(const KmeansGeom& g, const __nv_bfloat16* X, const float* init, float* cent,
                               const KmeansScratch& sc, cudaStream_t s) {
  const long long warps = (long long)g.BH * g.c_pad;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  kmeans_init_kernel<<<(unsigned)blocks, threads, 0, s>>>(g, X, init, cent, sc.cmma, sc.nrow, sc.arrive);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ assign
// CTA pairs: a cluster of two CTAs (the two SMs of a TPC) computes the
// distances of a unit of 256 tokens of one head to a chunk of <= 256
// centroids, one M = 256 tcgen05 MMA (.cta_group::2) per K-step of 16.  Each
// CTA stages its 128 token rows and half of the chunk's centroid rows and
// receives its rows' fp32 products in its own TMEM.  Few large MMAs matter
// here: M = 128 or N = 128 MMAs leave the tensor pipe half idle on issue and
// shared-memory reads, while one M = 256, N = 256 MMA per K-step keeps it
// busy.  Persistent: the pairs walk contiguous ranges of units over all
// heads.  Token tiles are triple-buffered (the next units stream in from HBM
// during the current one) and the centroid halves stream through a ring of
// K-blocks of 64 columns (TMA, 128-byte swizzle).  TMEM: 2 buffers x 256 fp32
// columns; epilogue group b reduces the chunks that land in buffer b, split
// between two halves of 4 warps that take the lower and upper half of the
// chunk's columns (16-column TMEM loads, the next in flight while one is
// reduced): the reduction waits on TMEM loads, so twice the warps keep twice
// the loads in flight.  One more K = 16 step of each chunk's MMA adds
// -||c||^2 / 2 (a block of ones in shared memory against the chunk's norm rows,
// both 32-byte swizzled), so TMEM holds x.c - ||c||^2 / 2 and the epilogue is
// a bare argmax with no per-column norm.  A unit's partial maxima merge
// through shared memory, the upper half into the lower, then group 1 into
// group 0.  Warps: 0
// centroid producer, 1 TMEM owner + MMA issuer (leader CTA), 2 token
// producer, 4 + 8h + 4b + q: group b, half h, TMEM lane quarter q.
namespace {
constexpr int kAssignThreads = 640;
constexpr int kAssignStages = 6;
constexpr int kAssignXBufs = 3;  // token tiles in flight

template <int D>
struct AssignSmem {
  static constexpr int kXBlocks = D / 64;                   // 64-column K-blocks of a token tile
  static constexpr int kXTileBytes = kXBlocks * 128 * 128;  // 128 rows x D bf16
  static constexpr int kStageBytes = 128 * 128;             // <= 128 centroid rows x 64 columns
  static constexpr int kX = 0;                              // token tile ring
  static constexpr int kStages = kX + kAssignXBufs * kXTileBytes;
  static constexpr int kMerge = kStages + kAssignStages * kStageBytes;  // [2 slots][128] (distance, index)
  static constexpr int kHMerge = kMerge + 2 * 128 * 8;                  // [group][2 slots][128] (distance, index)
  // ones block of the norm step: 128 rows x 32 B (1024-aligned)
  static constexpr int kOnes = (kHMerge + 4 * 128 * 8 + 1023) / 1024 * 1024;
  static constexpr int kBars = kOnes + 128 * 32;
  // c_full, c_empty [stages]; x_full, x_empty [x bufs]; t_full, t_empty, m_full, m_empty [2]; fin;
  // h_full, h_empty [group][2]
  static constexpr int kNumBars = 2 * kAssignStages + 2 * kAssignXBufs + 8 + 1 + 8;
  static constexpr int kMisc = kBars + kNumBars * 8;  // tmem base, abort flag
  static constexpr size_t bytes() { return 1024 + kMisc + 16; }
};
}  // namespace

// Next 256-token unit of a pair's range: (head, unit within the head).  The
// roles walk their units with this cursor rather than dividing a 64-bit unit
// index per unit, a long dependent chain for the single issuing threads.
__device__ __forceinline__ void next_unit(int& bh, int& pr, int uph) {
  if (++pr == uph) {
    pr = 0;
    ++bh;
  }
}

// Folds 16 columns of x.c - ||c||^2 / 2 into the running (best, best_j): the
// largest value is the smallest distance ||c||^2 - 2 x.c.  Argmax by a
// pairwise tree in which the right operand wins only when strictly larger,
// and the running maximum is replaced only by a strictly larger one, so ties
// keep the lowest index; padding centroids hold -inf and never win.
__device__ __forceinline__ void assign_argmax16(const float (&x)[16], int j0, float& best, int& best_j) {
  float m[8];
  int ix[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    ix[u] = x[2 * u + 1] > x[2 * u] ? 2 * u + 1 : 2 * u;
    m[u] = fmaxf(x[2 * u], x[2 * u + 1]);
  }
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1) {
#pragma unroll
    for (int k = 0; k < w; ++k) {
      const bool gt = m[2 * k + 1] > m[2 * k];
      ix[k] = gt ? ix[2 * k + 1] : ix[2 * k];
      m[k] = fmaxf(m[2 * k], m[2 * k + 1]);
    }
  }
  if (m[0] > best) {
    best = m[0];
    best_j = j0 + ix[0];
  }
}

template <int D>
__global__ void __launch_bounds__(kAssignThreads, 1)
    kmeans_assign_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                         const __grid_constant__ CUtensorMap tmap_n, KmeansGeom g, int32_t* __restrict__ assign) {
  using L = AssignSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* c_full = bars;  // leader's copy counts both CTAs' bytes
  uint64_t* c_empty = bars + kAssignStages;
  uint64_t* x_full = bars + 2 * kAssignStages;  // [x bufs] leader's copy counts both CTAs' bytes
  uint64_t* x_empty = x_full + kAssignXBufs;    // [x bufs]
  uint64_t* t_full = x_empty + kAssignXBufs;    // [2] per TMEM buffer
  uint64_t* t_empty = t_full + 2;               // [2] leader's copy, both CTAs' epilogue warps
  uint64_t* m_full = t_full + 4;                // [2] per merge slot
  uint64_t* m_empty = t_full + 6;               // [2]
  uint64_t* fin = t_full + 8;
  uint64_t* h_full = t_full + 9;    // [group * 2 + slot]
  uint64_t* h_empty = t_full + 13;  // [group * 2 + slot]
  float2* merge = reinterpret_cast<float2*>(smem + L::kMerge);
  float2* hmerge = reinterpret_cast<float2*>(smem + L::kHMerge);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int uph = (g.N + 255) / 256;  // 256-token units per head
  const long long total = (long long)g.BH * uph;
  const int npairs = gridDim.x / 2, pair = blockIdx.x / 2;
  const long long u0 = total * pair / npairs;
  const int nunits = (int)(total * (pair + 1) / npairs - u0);
  if (nunits <= 0) return;  // the same for both CTAs of the pair
  const int bh0 = (int)(u0 / uph), pr0 = (int)(u0 % uph);  // first unit
  const int nchunks = g.c_pad / g.chunk;
  const int half = g.chunk / 2;         // centroid rows per CTA per chunk
  const int kblocks = 2 * L::kXBlocks;  // hi blocks then lo blocks
  // A single chunk whose K-blocks all fit in the ring stays resident: it is
  // loaded once per head (an epoch) into stages 0..kblocks-1 instead of once
  // per unit, and the MMA issuer waits on it only when the head changes.
  const bool resident = nchunks == 1 && kblocks <= kAssignStages;
  // hi | lo along N: the resident chunk takes d / 64 stages, the hi rows in
  // the leader, the lo rows in the peer; TMEM column j is x.c_hi of centroid
  // j, column chunk + j its x.c_lo
  const bool hilo = resident && kmeans_hilo_n(g);
  const int rkb = hilo ? L::kXBlocks : kblocks;  // resident stages

  if (tid == 0) {
    for (int s = 0; s < kAssignStages; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 1);
    }
    for (int b = 0; b < kAssignXBufs; ++b) {
      mbar_init(&x_full[b], 1);
      mbar_init(&x_empty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], 16);  // one epilogue group: 8 warps x 2 CTAs
      mbar_init(&m_full[b], 4);
      mbar_init(&m_empty[b], 4);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&h_full[b], 4);
      mbar_init(&h_empty[b], 4);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  if (warp >= 4 && warp < 8) {
    // A operand of the norm step: bf16 ones at columns 0-2 and 8-10 of every
    // token row (the same 16 bytes in both halves of the 32-byte row)
    const uint32_t row = smem_u32(smem + L::kOnes) + (uint32_t)(tid - 128) * 32u;
    st_shared_v4(row, 0x3F803F80u, 0x00003F80u, 0u, 0u);
    st_shared_v4(row + 16, 0x3F803F80u, 0x00003F80u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers and TMEM of both CTAs ready before any cross-CTA traffic
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t x_base = smem_u32(smem + L::kX);
  const uint32_t st_base = smem_u32(smem + L::kStages);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------ centroid producer (both)
    prefetch_tmap(&tmap_c);
    int st = 0;
    bool ok = true;
    int ep = -1, cur_bh = -1;  // resident: epoch = head
    for (int i = 0, bh = bh0, pr = pr0; i < nunits && ok; ++i, next_unit(bh, pr, uph)) {
      if (resident) {
        if (bh == cur_bh) continue;
        cur_bh = bh;
        ++ep;
        // stages 0..rkb-1 the operand K-blocks, stage rkb the norm rows
        const int nr = hilo ? g.chunk : half;  // centroid rows per CTA
        const int row0 = hilo ? bh * g.c_pad : bh * g.c_pad + (int)rank * half;
        for (int kb = 0; kb <= rkb; ++kb) {
          if (ep >= 1 && !mbar_wait(&c_empty[kb], (ep - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&c_full[kb], 2 * nr * (kb < rkb ? 128 : 32));
          const uint32_t bar = mapa_shared(smem_u32(&c_full[kb]), 0);
          if (kb == rkb)
            tma_load_2d_pair(st_base + kb * L::kStageBytes, &tmap_n, hilo ? (int)rank * 16 : 0, row0, bar);
          else
            tma_load_2d_pair(st_base + kb * L::kStageBytes, &tmap_c, hilo ? (int)rank * g.d + kb * 64 : kb * 64,
                             row0, bar);
        }
        continue;
      }
      for (int c = 0; c < nchunks && ok; ++c) {
        // the chunk's operand K-blocks, then its norm rows
        for (int kb = 0; kb <= kblocks; ++kb, ++st) {
          const int s = st % kAssignStages;
          if (st >= kAssignStages && !mbar_wait(&c_empty[s], ((st / kAssignStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&c_full[s], 2 * half * (kb < kblocks ? 128 : 32));
          const int row0 = bh * g.c_pad + c * g.chunk + (int)rank * half;
          const uint32_t bar = mapa_shared(smem_u32(&c_full[s]), 0);
          if (kb == kblocks)
            tma_load_2d_pair(st_base + s * L::kStageBytes, &tmap_n, 0, row0, bar);
          else
            tma_load_2d_pair(st_base + s * L::kStageBytes, &tmap_c, kb * 64, row0, bar);
        }
      }
    }
  } else if (warp == 2 && lane == 0) {
    // --------------------------------------------- token producer (both)
    prefetch_tmap(&tmap_x);
    for (int i = 0, bh = bh0, pr = pr0; i < nunits; ++i, next_unit(bh, pr, uph)) {
      const int buf = i % kAssignXBufs;
      if (i >= kAssignXBufs && !mbar_wait(&x_empty[buf], ((i / kAssignXBufs) - 1) & 1, abort_flag)) break;
      const int row = bh * g.N + pr * 256 + (int)rank * 128;
      if (rank == 0) mbar_arrive_expect_tx(&x_full[buf], 2 * L::kXTileBytes);
      const uint32_t bar = mapa_shared(smem_u32(&x_full[buf]), 0);
      for (int kb = 0; kb < L::kXBlocks; ++kb)
        tma_load_2d_pair(x_base + buf * L::kXTileBytes + kb * 16384, &tmap_x, kb * 64, row, bar);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------- MMA (leader)
    const uint32_t idesc = umma_idesc_bf16(256, hilo ? 2 * g.chunk : g.chunk, false, false);
    // descriptors formed once: an operand's descriptor is the base one plus
    // its byte offset / 16 (the start-address field; no carry out of it, as
    // shared-memory offsets stay below 256 KB)
    const uint64_t adesc0 = umma_desc_sw128(x_base, 16, 1024);
    const uint64_t bdesc0 = umma_desc_sw128(st_base, 16, 1024);
    // norm step: the ones block against a stage of norm rows
    const uint64_t ones_desc = umma_desc_sw32(smem_u32(smem + L::kOnes));
    const uint64_t ndesc0 = umma_desc_sw32(st_base);
    int st = 0, gc = 0;  // stage counter, global chunk counter (TMEM buffer phases)
    bool ok = true;
    int ep = -1, cur_bh = -1;  // resident: epoch = head
    for (int i = 0, bh = bh0, pr = pr0; i < nunits && ok; ++i, next_unit(bh, pr, uph)) {
      const int buf = i % kAssignXBufs;
      if (!mbar_wait(&x_full[buf], (i / kAssignXBufs) & 1, abort_flag)) break;
      const uint64_t xdesc = adesc0 + (uint64_t)((buf * L::kXTileBytes) >> 4);
      if (resident) {
        const bool head_ends = i + 1 == nunits || pr + 1 == uph;
        const int b = gc & 1;
        if (gc >= 2 && !mbar_wait(&t_empty[b], ((gc >> 1) - 1) & 1, abort_flag)) break;
        if (bh != cur_bh) {
          cur_bh = bh;
          ++ep;
          for (int kb = 0; kb <= rkb && ok; ++kb)
            if (!mbar_wait(&c_full[kb], ep & 1, abort_flag)) ok = false;
          if (!ok) break;
        }
        tc_fence_after();
        if (hilo) {
#pragma unroll
          for (int kb = 0; kb < L::kXBlocks; ++kb)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ss_pair(tmem + (uint32_t)(b * 256), xdesc + (uint64_t)((kb * 16384 + k * 32) >> 4),
                                bdesc0 + (uint64_t)((kb * L::kStageBytes + k * 32) >> 4), idesc, (kb | k) != 0);
        } else {
#pragma unroll
          for (int kb = 0; kb < kblocks; ++kb) {
            const int xkb = kb % L::kXBlocks;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ss_pair(tmem + (uint32_t)(b * 256), xdesc + (uint64_t)((xkb * 16384 + k * 32) >> 4),
                                bdesc0 + (uint64_t)((kb * L::kStageBytes + k * 32) >> 4), idesc, (kb | k) != 0);
          }
        }
        umma_bf16_ss_pair(tmem + (uint32_t)(b * 256), ones_desc,
                          ndesc0 + (uint64_t)((rkb * L::kStageBytes) >> 4), idesc, 1u);
        if (head_ends)
          for (int kb = 0; kb <= rkb; ++kb) umma_commit_pair_mc(&c_empty[kb], 3);
        umma_commit_pair_mc(&t_full[b], 3);
        ++gc;
        umma_commit_pair_mc(&x_empty[buf], 3);
        continue;
      }
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
          const uint64_t sdesc = bdesc0 + (uint64_t)((s * L::kStageBytes) >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ss_pair(tmem + (uint32_t)(b * 256), xdesc + (uint64_t)((xkb * 16384 + k * 32) >> 4),
                              sdesc + (uint64_t)((k * 32) >> 4), idesc, (kb | k) != 0);
          umma_commit_pair_mc(&c_empty[s], 3);
        }
        if (!ok) break;
        {  // norm step
          const int s = st % kAssignStages;
          if (!mbar_wait(&c_full[s], (st / kAssignStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          umma_bf16_ss_pair(tmem + (uint32_t)(b * 256), ones_desc,
                            ndesc0 + (uint64_t)((s * L::kStageBytes) >> 4), idesc, 1u);
          umma_commit_pair_mc(&c_empty[s], 3);
          ++st;
        }
        umma_commit_pair_mc(&t_full[b], 3);
      }
      if (ok) umma_commit_pair_mc(&x_empty[buf], 3);
    }
    // drain: every issued MMA completes before TMEM is released
    umma_commit_pair(fin);
    mbar_wait_drain(fin, 0);
  } else if (warp >= 4) {
    // ------------------------------------------------- epilogue (both)
    const int ew = warp - 4;
    const int grp = (ew >> 2) & 1;         // TMEM buffer this warp reduces
    const int hf = ew >> 3;                // column half of the chunk
    const int r = (warp & 3) * 32 + lane;  // row of this CTA's tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((r & ~31) << 16);
    const uint32_t t_empty_lead = mapa_shared(smem_u32(&t_empty[grp]), 0);
    // this half's columns of a chunk, [h0, h1): multiples of 16, at most 128
    const int hcols = (g.chunk / 2 + 15) / 16 * 16;
    const int h0 = hf * hcols, h1 = min(g.chunk, h0 + hcols);
    const int ncol = h1 - h0;
    int gc = 0, hm = 0;  // global chunk counter, half merges of this group
    bool ok = true;
    for (int i = 0, bh = bh0, pr = pr0; i < nunits && ok; ++i, next_unit(bh, pr, uph)) {
      float best = -__int_as_float(0x7f800000);
      int best_j = 0;
      for (int c = 0; c < nchunks; ++c, ++gc) {
        const int b = gc & 1;
        if (b != grp) continue;
        if (!mbar_wait_warp(&t_full[b], (gc >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col0 = tmem + lane_off + (uint32_t)(b * 256 + h0);
        float va[16], vb[16];
        if (hilo) {
          // 16 centroids at a time: their hi and lo products, added
          for (int cb = 0; cb < ncol; cb += 16) {
            tmem_ld16(col0 + cb, va);
            tmem_ld16(col0 + g.chunk + cb, vb);
            tmem_wait_ld();
            pin_regs16(va);
            pin_regs16(vb);
#pragma unroll
            for (int e = 0; e < 16; ++e) va[e] += vb[e];
            assign_argmax16(va, h0 + cb, best, best_j);
          }
        }
        // 16-column groups, the next group's TMEM load in flight while one is
        // reduced (each wait covers the one load then outstanding)
        if (!hilo && ncol > 0) tmem_ld16(col0, va);
        for (int cb = 0; cb < ncol && !hilo; cb += 32) {
          tmem_wait_ld();
          pin_regs16(va);
          if (cb + 16 < ncol) tmem_ld16(col0 + cb + 16, vb);
          assign_argmax16(va, c * g.chunk + h0 + cb, best, best_j);
          if (cb + 16 < ncol) {
            tmem_wait_ld();
            pin_regs16(vb);
            if (cb + 32 < ncol) tmem_ld16(col0 + cb + 32, va);
            assign_argmax16(vb, c * g.chunk + h0 + cb + 16, best, best_j);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(t_empty_lead);
      }
      if (!ok) break;
      // with one chunk per unit the units alternate between the groups and
      // only the group that reduced this one holds its maximum
      if (nchunks == 1 && (gc - 1) % 2 != grp) continue;
      // the upper half hands its maximum to the lower half of the group; on
      // equal values the lower centroid index wins
      const int hs = grp * 2 + (hm & 1);
      float2* hslot = hmerge + hs * 128 + r;
      if (hf == 1) {
        if (hm >= 2 && !mbar_wait_warp(&h_empty[hs], ((hm >> 1) - 1) & 1, abort_flag)) break;
        *hslot = make_float2(best, __int_as_float(best_j));
        __syncwarp();
        if (lane == 0) mbar_arrive(&h_full[hs]);
        ++hm;
        continue;
      }
      if (!mbar_wait_warp(&h_full[hs], (hm >> 1) & 1, abort_flag)) break;
      {
        const float2 o = *hslot;
        const int oj = __float_as_int(o.y);
        if (o.x > best || (o.x == best && oj < best_j)) {
          best = o.x;
          best_j = oj;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&h_empty[hs]);
      ++hm;
      if (nchunks == 1) {
        const int tok = pr * 256 + (int)rank * 128 + r;
        if (tok < g.N) assign[(size_t)bh * g.N + tok] = best_j;
        continue;
      }
      // merge the two groups' maxima of this unit (slot i & 1)
      float2* slot = merge + (i & 1) * 128 + r;
      if (grp == 1) {
        if (i >= 2 && !mbar_wait_warp(&m_empty[i & 1], ((i >> 1) - 1) & 1, abort_flag)) break;
        *slot = make_float2(best, __int_as_float(best_j));
        __syncwarp();
        if (lane == 0) mbar_arrive(&m_full[i & 1]);
      } else {
        if (!mbar_wait_warp(&m_full[i & 1], (i >> 1) & 1, abort_flag)) break;
        const float2 o = *slot;
        const int oj = __float_as_int(o.y);
        const int jj = (o.x > best || (o.x == best && oj < best_j)) ? oj : best_j;
        __syncwarp();
        if (lane == 0) mbar_arrive(&m_empty[i & 1]);
        const int tok = pr * 256 + (int)rank * 128 + r;
        if (tok < g.N) assign[(size_t)bh * g.N + tok] = jj;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer is done with this CTA's barriers and TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

cudaError_t launch_kmeans_assign(const KmeansGeom& g, const CUtensorMap* tmap_x, const CUtensorMap* tmap_c,
                                 const CUtensorMap* tmap_n, int32_t* assign, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = (long long)g.BH * ((g.N + 255) / 256);
  int npairs = sms / 2;
  if (units < npairs) npairs = (int)units;
  if (npairs < 1) npairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * npairs);
  cfg.blockDim = dim3(kAssignThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (g.d == 128) {
    cfg.dynamicSmemBytes = AssignSmem<128>::bytes();
    cudaError_t e = cudaFuncSetAttribute(kmeans_assign_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cfg.dynamicSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kmeans_assign_kernel<128>, *tmap_x, *tmap_c, *tmap_n, g, assign);
  }
  cfg.dynamicSmemBytes = AssignSmem<64>::bytes();
  cudaError_t e = cudaFuncSetAttribute(kmeans_assign_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, kmeans_assign_kernel<64>, *tmap_x, *tmap_c, *tmap_n, g, assign);
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
// order, so the centroids do not depend on scheduling.  A thread's 16-byte
// chunks of its slot's rows are fetched with cp.async into a private ring
// of kUpdDepth shared-memory entries, so kUpdDepth rows per slot are in
// flight without holding registers; a thread reads only entries it copied,
// so the ring needs no barrier, only cp.async.wait_group.
constexpr int kUpdDepth = 8;  // rows in flight per slot


template <int kUpdThreads>
__global__ void __launch_bounds__(kUpdThreads)
    kmeans_update_kernel(KmeansGeom g, const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm,
                         const int32_t* __restrict__ offsets, float* __restrict__ cent,
                         __nv_bfloat16* __restrict__ cmma, __nv_bfloat16* __restrict__ nrows,
                         float* __restrict__ partial, int32_t* __restrict__ arrive,
                         const int4* __restrict__ pmap, int part_slots) {
  __shared__ __align__(16) uint4 ring[kUpdDepth][kUpdThreads];  // later the slot partial sums
  __shared__ int rows_s[kUpdRows];  // the piece's token indices
  __shared__ float red[32];
  __shared__ int s_c, s_piece, s_np, s_base, s_last;
  const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int32_t* off = offsets + (size_t)bh * (g.C + 1);

  // (cluster, piece) of this CTA: entry blockIdx.x of the head's piece map
  if (tid == 0) {
    const int4 e = pmap[(size_t)bh * gridDim.x + blockIdx.x];
    s_c = e.x;
    s_piece = e.y;
    s_np = e.z;
    s_base = e.w;
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
  for (int p = plo + tid; p < phi; p += kUpdThreads) rows_s[p - plo] = prow[p];
  __syncthreads();
  const __nv_bfloat16* xh = X + (size_t)bh * g.N * g.d + ch * 8;
  // this slot's rows: plo + slot + slots * k, k < nk, added in that order
  const int nk = phi - plo > slot ? (phi - plo - slot + slots - 1) / slots : 0;
  auto issue = [&](int k) {
    const int src = rows_s[slot + slots * k];
    const bool ok = src >= 0 && src < g.N;
    if (!ok) raise_error(kErrIndex);
    cp_async_16(smem_u32(&ring[k % kUpdDepth][tid]), xh + (size_t)(ok ? src : 0) * g.d, ok ? 16u : 0u);
  };
#pragma unroll
  for (int k = 0; k < kUpdDepth; ++k) {
    if (k < nk) issue(k);
    cp_async_commit();  // one group per row, empty past the end
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int k = 0; k < nk; ++k) {
    cp_async_wait<kUpdDepth - 1>();  // row k's group is the oldest of the last kUpdDepth
    const uint4 raw = ring[k % kUpdDepth][tid];
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
    // the entry is refilled only after its value was consumed above
    if (k + kUpdDepth < nk) issue(k + kUpdDepth);
    cp_async_commit();
  }
  cp_async_wait_all();
  __syncthreads();  // every ring read done: the ring becomes the slot sums
  float* part = reinterpret_cast<float*>(&ring[0][0]);
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
  if (wid == 0) {
    float tot = 0.f;
    for (int w = 0; w < (g.d + 31) / 32; ++w) tot += red[w];
    write_norm_row(tot, nrows + ((size_t)bh * g.c_pad + c) * kNormCols, lane);
  }
}

cudaError_t launch_kmeans_update(const KmeansGeom& g, const __nv_bfloat16* X, const int32_t* perm,
                                 const int32_t* offsets, float* cent, const KmeansScratch& sc, cudaStream_t s) {
  // at most C + N/R pieces per head (every cluster adds at most one piece
  // beyond n/R); CTAs past a head's last piece return at once.  Clusters of a
  // few hundred rows take 128 threads: a CTA's time is then mostly the
  // latency of its dependent loads (offsets, permutation, rows), and smaller
  // CTAs keep more of those chains in flight per SM.
  dim3 grid(kmeans_update_grid(g), g.BH);
  if ((long long)g.N < 512LL * g.C)
    kmeans_update_kernel<128><<<grid, 128, 0, s>>>(g, X, perm, offsets, cent, sc.cmma, sc.nrow, sc.partial,
                                                   sc.arrive, sc.pmap, kmeans_part_slots(g));
  else
    kmeans_update_kernel<256><<<grid, 256, 0, s>>>(g, X, perm, offsets, cent, sc.cmma, sc.nrow, sc.partial,
                                                   sc.arrive, sc.pmap, kmeans_part_slots(g));
  return cudaGetLastError();
}

}  // namespace ig
