// Semantic permutation (InstaGen abstract: tokens are reordered by cluster so
// the attention matrix becomes block structured; Figure 3 (d): a query group
// attends to one common key list, which makes the work dense tiles).  A stable
// counting sort puts every cluster in a contiguous range of slots, and a row
// gather copies K and V into that order with 128-bit coalesced loads and
// stores.
#include "internal.cuh"
#include "ptx.cuh"

#include <cooperative_groups.h>
#include <cuda_bf16.h>

namespace ig {

// --------------------------------------------------------- counting sort
// One thread-block cluster of S CTAs per head (S <= 16); CTA r owns the r-th
// of S contiguous token ranges, and warp w of it a contiguous sub-range.
// Phase 1 counts every warp's range per cluster; the CTA totals are exchanged
// through distributed shared memory, giving every CTA the global cluster
// starts and the number of earlier tokens of each cluster in lower-ranked
// CTAs; phase 3 walks each warp range in order (32 tokens at a time, ranks
// inside a step from __match_any_sync), so equal clusters keep ascending
// token index.  The first kSortRegs steps of a warp's range stay in registers
// from phase 1 to phase 3 (all their loads in flight at once; the ordered walk
// then waits on no memory); longer ranges read the rest again.  The sort is a
// single launch and needs no global scratch.  The ordered walk is a chain of
// dependent steps per warp, so when every head's cluster fits the device at
// once, a head is spread over 16 or else 12 CTAs (non-portable cluster sizes)
// with 24 or 32 register-held steps and 4 CTAs per SM, which shortens each
// warp's chain; otherwise over 8 CTAs with 40 steps and 3 CTAs per SM.
constexpr int kSortMaxCtas = 16;
constexpr int kSortPortableCtas = 8;
constexpr int kSortUnroll = 4;
constexpr int kSortMaxWarps = 8;   // 256 threads per CTA

template <int kSortRegs, int kMinBlocks>  // 32-token steps per warp held in registers; CTAs per SM
__global__ void __launch_bounds__(kSortMaxWarps * 32, kMinBlocks)
    count_sort_kernel(const int32_t* __restrict__ assign, int N, int C, int32_t* __restrict__ perm,
                                  int32_t* __restrict__ offsets, int4* __restrict__ pmap, int pgrid) {
  extern __shared__ int sort_smem[];  // cnt [nwarps][C], ctot [C], before [C], base [C+1]
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int S = (int)cluster.num_blocks();
  const int r = (int)cluster.block_rank();
  const int nwarps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int32_t* a = assign + (size_t)bh * N;
  int* cnt = sort_smem;
  int* ctot = cnt + nwarps * C;
  int* before = ctot + C;
  int* base = before + C;
  for (int i = threadIdx.x; i < nwarps * C; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int q0 = (int)((long long)N * r / S), q1 = (int)((long long)N * (r + 1) / S);
  const int seg = (q1 - q0 + nwarps - 1) / nwarps;
  const int s0 = min(q1, q0 + warp * seg), s1 = min(q1, s0 + seg);
  const int sreg = min(s1, s0 + 32 * kSortRegs);  // end of the register-held part
  int vr[kSortRegs];
#pragma unroll
  for (int k = 0; k < kSortRegs; ++k) {
    const int i = s0 + 32 * k + lane;
    vr[k] = i < sreg ? a[i] : -1;
  }
#pragma unroll
  for (int k = 0; k < kSortRegs; ++k) {
    if (s0 + 32 * k + lane < sreg) {
      if (vr[k] >= 0 && vr[k] < C)
        atomicAdd(&cnt[warp * C + vr[k]], 1);
      else
        raise_error(kErrIndex);
    }
  }
  for (int i0 = sreg + lane; i0 < s1; i0 += 32 * kSortUnroll) {
    int v[kSortUnroll];
#pragma unroll
    for (int u = 0; u < kSortUnroll; ++u) v[u] = (i0 + 32 * u < s1) ? a[i0 + 32 * u] : 0;
#pragma unroll
    for (int u = 0; u < kSortUnroll; ++u) {
      if (i0 + 32 * u >= s1) break;
      if (v[u] >= 0 && v[u] < C)
        atomicAdd(&cnt[warp * C + v[u]], 1);
      else
        raise_error(kErrIndex);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    int t = 0;
    for (int w = 0; w < nwarps; ++w) t += cnt[w * C + c];
    ctot[c] = t;
  }
  cluster.sync();  // every CTA's totals visible to the cluster
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    int all = 0, bef = 0;
    for (int q = 0; q < S; ++q) {
      const int v = cluster.map_shared_rank(ctot, q)[c];
      all += v;
      if (q < r) bef += v;
    }
    base[c] = all;
    before[c] = bef;
  }
  cluster.sync();  // no remote reads after this point
  // exclusive prefix of the cluster totals (one warp, chunks of 32)
  if (warp == 0) {
    int run = 0;
    for (int c0 = 0; c0 < C; c0 += 32) {
      const int c = c0 + lane;
      const int tot = c < C ? base[c] : 0;
      int incl = tot;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (c < C) base[c] = run + incl - tot;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) base[C] = run;
  }
  __syncthreads();
  if (r == 0)
    for (int c = threadIdx.x; c <= C; c += blockDim.x) offsets[(size_t)bh * (C + 1) + c] = base[c];
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    int run = base[c] + before[c];
    for (int w = 0; w < nwarps; ++w) {
      const int t = cnt[w * C + c];
      cnt[w * C + c] = run;
      run += t;
    }
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  int32_t* pout = perm + (size_t)bh * N;
  // one 32-token step in token order: lanes of equal cluster ranked by lane
  auto place = [&](int c, int i) {
    if (c >= C || c < 0) c = -1;
    const unsigned same = __match_any_sync(0xffffffffu, c);
    const int rank = __popc(same & lt_mask);
    int pos = 0;
    if (c >= 0) pos = cnt[warp * C + c] + rank;
    __syncwarp();
    if (c >= 0 && rank == 0) cnt[warp * C + c] += __popc(same);
    __syncwarp();
    if (c >= 0) pout[pos] = i;
  };
#pragma unroll
  for (int k = 0; k < kSortRegs; ++k) {
    const int i0 = s0 + 32 * k;
    if (i0 >= sreg) break;  // warp-uniform
    place(i0 + lane < sreg ? vr[k] : -1, i0 + lane);
  }
  int nxt = (sreg + lane < s1) ? a[sreg + lane] : -1;
  for (int i0 = sreg; i0 < s1; i0 += 32) {
    const int i = i0 + lane;
    const int c = nxt;
    nxt = (i + 32 < s1) ? a[i + 32] : -1;  // next step's load in flight
    place(c, i);
  }
  if (pmap != nullptr && r == 0) {
    // The centroid update's piece map of this head, from the cluster sizes:
    // exclusive prefixes over the clusters of their piece counts and of the
    // pieces of multi-piece clusters (block-wide: a range of clusters per
    // thread, warp scans, then the warp totals in order).
    __shared__ int s_scan[2 * kSortMaxWarps];
    const int nthr = blockDim.x;
    const int per = (C + nthr - 1) / nthr;
    const int c0 = min((int)threadIdx.x * per, C), c1 = min(c0 + per, C);
    int np = 0, mp = 0;
    for (int c = c0; c < c1; ++c) {
      const int k = update_pieces(base[c + 1] - base[c]);
      np += k;
      if (k > 1) mp += k;
    }
    int npi = np, mpi = mp;
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, npi, o), y = __shfl_up_sync(0xffffffffu, mpi, o);
      if (lane >= o) {
        npi += x;
        mpi += y;
      }
    }
    if (lane == 31) {
      s_scan[warp] = npi;
      s_scan[kSortMaxWarps + warp] = mpi;
    }
    __syncthreads();
    int p0 = npi - np, m0 = mpi - mp, total = 0;
    for (int w = 0; w < nwarps; ++w) {
      if (w < warp) {
        p0 += s_scan[w];
        m0 += s_scan[kSortMaxWarps + w];
      }
      total += s_scan[w];
    }
    int4* pm = pmap + (size_t)bh * pgrid;
    for (int c = c0; c < c1; ++c) {
      const int k = update_pieces(base[c + 1] - base[c]);
      for (int q = 0; q < k && p0 + q < pgrid; ++q) pm[p0 + q] = make_int4(c, q, k, m0);
      p0 += k;
      if (k > 1) m0 += k;
    }
    for (int t = total + (int)threadIdx.x; t < pgrid; t += nthr) pm[t] = make_int4(-1, 0, 0, 0);
  }
}

cudaError_t launch_count_sort(const int32_t* assign, int BH, int N, int C, int32_t* perm, int32_t* offsets,
                              int4* pmap, int pgrid, cudaStream_t s) {
  // one CTA per 4096 tokens of a head, up to a cluster of 8 (or 12 or 16, see
  // above); as many warps (<= kSortMaxWarps) as fit 160 KB of per-warp counters
  int S = (N + 4095) / 4096;
  S = S < 1 ? 1 : (S > kSortMaxCtas ? kSortMaxCtas : S);
  int nwarps = (int)((160 * 1024) / ((size_t)C * 4));
  nwarps = nwarps < 1 ? 1 : (nwarps > kSortMaxWarps ? kSortMaxWarps : nwarps);
  const size_t sm = ((size_t)nwarps * C + 3 * (size_t)C + 1) * sizeof(int);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(nwarps * 32);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the largest of 16 and 12 CTAs per head whose clusters all fit the device
  // at once, with enough register-held steps for a warp's range
  for (int Sx = kSortMaxCtas; Sx > kSortPortableCtas && S > kSortPortableCtas; Sx -= 4) {
    const int Su = S < Sx ? S : Sx;
    const int steps = (int)(((long long)N + (long long)Su * nwarps * 32 - 1) / ((long long)Su * nwarps * 32)) + 1;
    auto* kx = steps <= 24 ? count_sort_kernel<24, 4> : count_sort_kernel<32, 4>;
    cfg.gridDim = dim3(Su, BH);
    attr[0].val.clusterDim.x = Su;
    int active = 0;
    if (cudaFuncSetAttribute(kx, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) == cudaSuccess &&
        cudaFuncSetAttribute(kx, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaOccupancyMaxActiveClusters(&active, kx, &cfg) == cudaSuccess && active >= BH && steps <= 32)
      return cudaLaunchKernelEx(&cfg, kx, assign, N, C, perm, offsets, pmap, pgrid);
    cudaGetLastError();  // clear a refusal; a smaller size follows
  }
  S = S > kSortPortableCtas ? kSortPortableCtas : S;
  auto* k8 = count_sort_kernel<40, 3>;
  cudaError_t e = cudaFuncSetAttribute(k8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(S, BH);
  attr[0].val.clusterDim.x = S;
  return cudaLaunchKernelEx(&cfg, k8, assign, N, C, perm, offsets, pmap, pgrid);
}

// ---------------------------------------------------------------- gather
// Y[bh, p, :] = X[bh, perm[bh, p], :] for one or two tensors; each thread moves
// 16 bytes, consecutive threads move consecutive chunks of a row.  A tensor
// whose `to_f16` flag is set is converted from bf16 to fp16 on the way
// (values beyond the fp16 range are saturated and reported).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
  uint4 out;
  uint32_t* o = reinterpret_cast<uint32_t*>(&out);
  bool over = false;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    over |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
    f.x = fminf(fmaxf(f.x, -65504.f), 65504.f);
    f.y = fminf(fmaxf(f.y, -65504.f), 65504.f);
    o[e] = pack_f16x2(f.x, f.y);
  }
  if (over) raise_error(kErrRange);
  return out;
}

__global__ void gather_rows_kernel(const uint4* __restrict__ X0, const uint4* __restrict__ X1,
                                   const int32_t* __restrict__ perm, long long rows, int N, int cpr,
                                   uint4* __restrict__ Y0, uint4* __restrict__ Y1, int f16_0, int f16_1) {
  const long long total = rows * cpr;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const long long row = g / cpr;
    const int ch = (int)(g - row * cpr);
    const long long bh = row / N;
    const int src = perm[row];
    if (src < 0 || src >= N) {
      raise_error(kErrIndex);
      continue;
    }
    const long long si = (bh * N + src) * cpr + ch;
    const uint4 v0 = X0[si];
    Y0[g] = f16_0 ? bf16x8_to_f16x8(v0) : v0;
    if (X1) {
      const uint4 v1 = X1[si];
      Y1[g] = f16_1 ? bf16x8_to_f16x8(v1) : v1;
    }
  }
}

cudaError_t launch_gather_rows(const __nv_bfloat16* X0, const __nv_bfloat16* X1, const int32_t* perm, int BH,
                               int N, int d, void* Y0, void* Y1, bool f16_0, bool f16_1, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cpr = d * 2 / 16;
  const long long rows = (long long)BH * N;
  const long long work = rows * cpr;
  const int threads = 512;
  long long blocks = (work + threads - 1) / threads;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  gather_rows_kernel<<<(unsigned)blocks, threads, 0, s>>>(
      reinterpret_cast<const uint4*>(X0), reinterpret_cast<const uint4*>(X1), perm, rows, N, cpr,
      reinterpret_cast<uint4*>(Y0), reinterpret_cast<uint4*>(Y1), f16_0 ? 1 : 0, f16_1 ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(int* value, cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  *value = v;
  return e;
}

}  // namespace ig
