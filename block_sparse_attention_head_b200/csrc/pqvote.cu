// Product-quantised per-query voting: the selection rule of the InstaGen
// abstract (thelatestinai.com paper page and the paper-reading aggregator
// page: queries and keys are product-quantised so that a block score is cheap
// for every query rather than only for the cluster centroid; each query votes
// for its top blocks and the cluster attends to the blocks with the most
// votes).  An alternative to ranking key groups by centroid scores (Figure 3
// (b)-(c)); pi and the sample keep the centroid scores.
//
// Parameters the pages leave open, as read here: subspaces of 8 consecutive
// dimensions (M = d/8) with 16 codewords each, one codebook per side and
// head, trained by 5 Lloyd iterations on that side's group centroids (first
// min(16, C) centroids as the start; ties to the lowest codeword; an empty
// codeword keeps its value); a query token is encoded against the query
// codebook and a key group by its centroid against the key codebook; the
// block score is the sum over subspaces (m ascending, fp32 from +0) of the
// inner product of the two codewords (an fma chain over the 8 coordinates);
// each query votes for the prefix of its ranking (non-empty groups by score
// descending, lowest index first on ties) that the exact-set budget rule
// takes: rank 0 always, then while the running key count stays <= E.
// Every step is a correctly rounded fp32 operation in a fixed order.
#include "internal.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace ig {

namespace {
constexpr int kPqSub = 8;
constexpr int kPqKc = 16;
constexpr int kPqIters = 5;
constexpr int kPqCbThreads = 128;
constexpr int kPqVoteThreads = 256;
constexpr int kPqChunk = 128;  // queries per CTA of the vote kernel

__device__ __forceinline__ float pq_dist8(const float* x, const float* c) {
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < kPqSub; ++e) {
    const float t = __fsub_rn(x[e], c[e]);
    acc = __fmaf_rn(t, t, acc);
  }
  return acc;
}

// nearest of kc codewords (rows of 8 floats), ties to the lowest index
__device__ __forceinline__ int pq_nearest(const float* x, const float* cb, int kc) {
  int best = 0;
  float bd = pq_dist8(x, cb);
  for (int c = 1; c < kc; ++c) {
    const float dd = pq_dist8(x, cb + c * kPqSub);
    if (dd < bd) {
      bd = dd;
      best = c;
    }
  }
  return best;
}
}  // namespace

// Codebook of subspace m of one side of one head: grid (M, 2, BH); side 0 =
// queries (points cq [C = Cq]), side 1 = keys (points ck [C = Ck]).  The
// assignments live in shared memory; a codeword coordinate is updated by one
// thread summing its members in point order.  Side 1 also writes the key
// groups' codes.
__global__ void __launch_bounds__(kPqCbThreads)
    pq_codebook_kernel(PqArgs a) {
  extern __shared__ __align__(16) uint8_t pq_sm[];
  uint8_t* asg = pq_sm;  // [C]
  __shared__ float cb[kPqKc * kPqSub];
  const int m = blockIdx.x, side = blockIdx.y, bh = blockIdx.z, tid = threadIdx.x;
  const int C = side ? a.Ck : a.Cq, d = a.d;
  const float* P = (side ? a.ck + (size_t)bh * a.Ck * d : a.cq + (size_t)bh * a.Cq * d) + m * kPqSub;
  const int kc = C < kPqKc ? C : kPqKc;
  for (int t = tid; t < kPqKc * kPqSub; t += kPqCbThreads) {
    const int c = t / kPqSub, e = t % kPqSub;
    cb[t] = c < kc ? P[(size_t)c * d + e] : 0.0f;
  }
  __syncthreads();
  for (int it = 0; it < kPqIters; ++it) {
    for (int p = tid; p < C; p += kPqCbThreads) {
      float x[kPqSub];
#pragma unroll
      for (int e = 0; e < kPqSub; ++e) x[e] = P[(size_t)p * d + e];
      asg[p] = (uint8_t)pq_nearest(x, cb, kc);
    }
    __syncthreads();
    float nv = 0.0f;
    bool upd = false;
    if (tid < kc * kPqSub) {
      const int c = tid / kPqSub, e = tid % kPqSub;
      float sum = 0.0f;
      int n = 0;
      for (int p = 0; p < C; ++p)
        if (asg[p] == c) {
          sum = __fadd_rn(sum, P[(size_t)p * d + e]);
          ++n;
        }
      if (n > 0) {
        nv = __fdiv_rn(sum, (float)n);
        upd = true;
      }
    }
    __syncthreads();
    if (upd) cb[tid] = nv;
    __syncthreads();
  }
  float* out = a.codebooks + (((size_t)bh * 2 + side) * (d / kPqSub) + m) * kPqKc * kPqSub;
  for (int t = tid; t < kPqKc * kPqSub; t += kPqCbThreads) out[t] = cb[t];
  if (side == 1) {
    const int M = d / kPqSub;
    for (int p = tid; p < C; p += kPqCbThreads) {
      float x[kPqSub];
#pragma unroll
      for (int e = 0; e < kPqSub; ++e) x[e] = P[(size_t)p * d + e];
      a.kcodes[((size_t)bh * a.Ck + p) * M + m] = (uint8_t)pq_nearest(x, cb, kc);
    }
  }
}

namespace {
__device__ __forceinline__ uint32_t pq_float_order(float s) {
  if (s == 0.0f) s = 0.0f;
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
}  // namespace

// Votes of a chunk of at most kPqChunk queries of one query group: grid
// (chunks, BH), 8 warps, one query per warp at a time; the chunk's votes are
// added to the group's (integer atomics: the totals do not depend on order),
// so a large group is spread over many CTAs.
template <int KPL>
__global__ void __launch_bounds__(kPqVoteThreads) pq_votes_kernel(PqArgs a) {
  extern __shared__ __align__(16) uint8_t pq_sm[];
  const int M = a.d / kPqSub, Ck = a.Ck;
  float* T = reinterpret_cast<float*>(pq_sm);      // [M][16][16] codeword inner products
  float* cbq = T + M * kPqKc * kPqKc;              // [M][16][8] query codebook
  // the two int arrays are padded to a multiple of 4 entries so that the
  // code rows after them start on a 16-byte boundary (16- or 8-byte loads)
  const int Ck4 = (Ck + 3) & ~3;
  int* wsz = reinterpret_cast<int*>(cbq + M * kPqKc * kPqSub);  // [Ck4] key-group sizes
  int* votes_s = wsz + Ck4;                        // [Ck4]
  uint8_t* kc_s = reinterpret_cast<uint8_t*>(votes_s + Ck4);  // [Ck][M] key-group codes
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ int s_work[2];  // query group, chunk within it
  const int32_t* qoff = a.q_offsets + (size_t)bh * (a.Cq + 1);
  if (warp == 0) {
    const int t_glob = blockIdx.x;
    int run = 0, found_g = -1, found_c = 0;
    for (int c0 = 0; c0 < a.Cq && found_g < 0; c0 += 32) {
      const int c = c0 + lane;
      const int nc = (c < a.Cq) ? (max(qoff[c + 1] - qoff[c], 0) + kPqChunk - 1) / kPqChunk : 0;
      int incl = nc;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = run + incl - nc;
      const bool mine = nc > 0 && t_glob >= excl && t_glob < excl + nc;
      const unsigned hit = __ballot_sync(0xffffffffu, mine);
      if (hit) {
        const int src = __ffs(hit) - 1;
        found_g = __shfl_sync(0xffffffffu, c, src);
        found_c = __shfl_sync(0xffffffffu, t_glob - excl, src);
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_work[0] = found_g;
      s_work[1] = found_c;
    }
  }
  __syncthreads();
  const int i = s_work[0];
  if (i < 0) return;  // chunk index beyond this head's chunks
  const float* cbh = a.codebooks + (size_t)bh * 2 * M * kPqKc * kPqSub;
  for (int t = tid; t < M * kPqKc * kPqKc; t += kPqVoteThreads) {
    const int m = t / (kPqKc * kPqKc), qa = (t / kPqKc) % kPqKc, kb = t % kPqKc;
    const float* x = cbh + ((size_t)m * kPqKc + qa) * kPqSub;
    const float* y = cbh + ((size_t)(M + m) * kPqKc + kb) * kPqSub;
    float acc = 0.0f;
#pragma unroll
    for (int e = 0; e < kPqSub; ++e) acc = __fmaf_rn(x[e], y[e], acc);
    T[t] = acc;
  }
  for (int t = tid; t < M * kPqKc * kPqSub; t += kPqVoteThreads) cbq[t] = cbh[t];
  const int32_t* koff = a.k_offsets + (size_t)bh * (Ck + 1);
  for (int j = tid; j < Ck; j += kPqVoteThreads) {
    wsz[j] = max(koff[j + 1] - koff[j], 0);
    votes_s[j] = 0;
  }
  for (int t = tid; t < Ck * M; t += kPqVoteThreads) kc_s[t] = a.kcodes[(size_t)bh * Ck * M + t];
  __syncthreads();

  const int kcq = a.Cq < kPqKc ? a.Cq : kPqKc;
  const int qlo = qoff[i] + s_work[1] * kPqChunk, qhi = min(qoff[i + 1], qlo + kPqChunk);
  const long long E = a.E;
  // A query's votes depend only on its codes: each warp keeps the last code
  // vector and the key groups it voted for (bit k of a lane's mask: group
  // lane + 32k), and a run of queries with equal codes is added as a count.
  bool has_prev = false;
  unsigned long long prev_cv = 0ull;
  unsigned long long vmask = 0ull;  // KPL <= 64 bits
  int run = 0;
  auto flush = [&]() {
    if (run > 0) {
#pragma unroll
      for (int k = 0; k < KPL; ++k)
        if ((vmask >> k) & 1ull) atomicAdd(&votes_s[lane + 32 * k], run);
    }
    run = 0;
  };
  for (int slot = qlo + warp; slot < qhi; slot += kPqVoteThreads / 32) {
    const int tok = a.q_perm[(size_t)bh * a.N + slot];
    if (tok < 0 || tok >= a.N) {  // the same for every lane
      if (lane == 0) raise_error(kErrIndex);
      continue;
    }
    // encode: lane m < M takes subspace m of the query
    int code = 0;
    if (lane < M) {
      const uint4 raw = *reinterpret_cast<const uint4*>(a.Q + ((size_t)bh * a.N + tok) * a.d + kPqSub * lane);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float x[kPqSub];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
      }
      code = pq_nearest(x, cbq + lane * kPqKc * kPqSub, kcq);
    }
    int am[16];
    unsigned long long cv = 0ull;  // the codes, 4 bits each
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      am[m] = __shfl_sync(0xffffffffu, code, m);
      if (m < M) cv |= (unsigned long long)am[m] << (4 * m);
    }
    if (has_prev && cv == prev_cv) {
      ++run;
      continue;
    }
    flush();
    // score order of this lane's key groups j = lane + 32k (weight 0: empty or absent)
    uint32_t so[KPL];
    int wk[KPL];
    uint32_t top = 0u;
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      const int j = lane + 32 * k;
      so[k] = 0u;
      wk[k] = 0;
      if (j < Ck && wsz[j] > 0) {
        // the group's M codes in one 16-byte (d = 128) or 8-byte (d = 64) load
        uint4 cw = make_uint4(0u, 0u, 0u, 0u);
        if (M == 16) {
          cw = *reinterpret_cast<const uint4*>(kc_s + j * 16);
        } else {
          const uint2 c2 = *reinterpret_cast<const uint2*>(kc_s + j * 8);
          cw.x = c2.x;
          cw.y = c2.y;
        }
        const uint32_t cwv[4] = {cw.x, cw.y, cw.z, cw.w};
        float sc = 0.0f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < M) sc = __fadd_rn(sc, T[(m * kPqKc + am[m]) * kPqKc + ((cwv[m >> 2] >> (8 * (m & 3))) & 0xFFu)]);
        so[k] = pq_float_order(sc);  // >= 0x007FFFFF for a finite score
        wk[k] = wsz[j];
        top = max(top, so[k]);
      }
    }
    // Budget prefix in rank order (score descending, then lower j): the
    // groups strictly above the boundary score level (binary search for the
    // smallest level u with W(score order >= u) <= E), then the groups at the
    // boundary level in j order while they fit (rank 0 always).
    auto W_ge = [&](uint32_t u) -> long long {
      unsigned w = 0u;
#pragma unroll
      for (int k = 0; k < KPL; ++k) w += so[k] >= u ? (unsigned)wk[k] : 0u;  // empty: weight 0
      return (long long)__reduce_add_sync(0xffffffffu, w);
    };
    vmask = 0ull;
    if (W_ge(1u) <= E) {  // every group fits
#pragma unroll
      for (int k = 0; k < KPL; ++k)
        if (wk[k] > 0) vmask |= 1ull << k;
    } else {
      uint32_t lo = 1u, hi = __reduce_max_sync(0xffffffffu, top) + 1u;  // W(>= lo) > E >= W(>= hi) = 0
      long long w_hi = 0;
#pragma unroll 1
      while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const long long w = W_ge(mid);
        if (w > E) {
          lo = mid;
        } else {
          hi = mid;
          w_hi = w;
        }
      }
#pragma unroll
      for (int k = 0; k < KPL; ++k)
        if (wk[k] > 0 && so[k] >= hi) vmask |= 1ull << k;
      // boundary level lo, in ascending j
      long long acc = w_hi;
      bool stop = false;
#pragma unroll
      for (int k = 0; k < KPL; ++k) {
        unsigned tied = __ballot_sync(0xffffffffu, wk[k] > 0 && so[k] == lo);
        while (tied != 0u && !stop) {
          const int src = __ffs(tied) - 1;
          tied &= tied - 1u;
          const long long w = __shfl_sync(0xffffffffu, wk[k], src);
          if (acc == 0 || acc + w <= E) {  // acc == 0: nothing ranks above, rank 0 is kept
            acc += w;
            if (lane == src) vmask |= 1ull << k;
          } else {
            stop = true;
          }
        }
        if (stop) break;
      }
    }
    prev_cv = cv;
    has_prev = true;
    run = 1;
  }
  flush();
  __syncthreads();
  int32_t* vout = a.votes + ((size_t)bh * a.Cq + i) * Ck;
  for (int j = tid; j < Ck; j += kPqVoteThreads)
    if (votes_s[j] != 0) atomicAdd(vout + j, votes_s[j]);
}

size_t pq_scratch_bytes(int BH, int d, int Ck) {
  const size_t M = (size_t)d / kPqSub;
  const size_t cb = (size_t)BH * 2 * M * kPqKc * kPqSub * sizeof(float);
  const size_t codes = (size_t)BH * Ck * M;
  return (cb + 255) / 256 * 256 + (codes + 255) / 256 * 256;
}

cudaError_t launch_pq_votes(const PqArgs& a0, void* scratch, cudaStream_t s) {
  PqArgs a = a0;
  const int M = a.d / kPqSub;
  a.codebooks = reinterpret_cast<float*>(scratch);
  const size_t cb = (size_t)a.BH * 2 * M * kPqKc * kPqSub * sizeof(float);
  a.kcodes = reinterpret_cast<uint8_t*>(scratch) + (cb + 255) / 256 * 256;
  cudaError_t z = cudaMemsetAsync(a.votes, 0, (size_t)a.BH * a.Cq * a.Ck * sizeof(int32_t), s);
  if (z != cudaSuccess) return z;
  const int cmax = a.Cq > a.Ck ? a.Cq : a.Ck;
  pq_codebook_kernel<<<dim3(M, 2, a.BH), kPqCbThreads, (size_t)cmax, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t Ck4 = ((size_t)a.Ck + 3) & ~(size_t)3;
  const size_t sm = (size_t)M * kPqKc * kPqKc * 4 + (size_t)M * kPqKc * kPqSub * 4 + Ck4 * 8 + (size_t)a.Ck * M;
  const int kpl = (a.Ck + 31) / 32;
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (r != cudaSuccess) return r;
    // chunks per head <= ceil(N / chunk) + Cq (one ragged chunk per group)
    kern<<<dim3((a.N + kPqChunk - 1) / kPqChunk + a.Cq, a.BH), kPqVoteThreads, sm, s>>>(a);
    return cudaGetLastError();
  };
  if (kpl <= 4) return go(pq_votes_kernel<4>);
  if (kpl <= 8) return go(pq_votes_kernel<8>);
  if (kpl <= 16) return go(pq_votes_kernel<16>);
  if (kpl <= 32) return go(pq_votes_kernel<32>);
  return go(pq_votes_kernel<64>);
}

}  // namespace ig
