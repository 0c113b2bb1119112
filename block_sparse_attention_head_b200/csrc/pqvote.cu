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
  extern __shared__ uint8_t pq_sm[];
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

// Votes of query group i of head bh: grid (Cq, BH), 8 warps, one query per
// warp at a time.  A query's keys are ranked by the 44-bit key (score order
// << 12 | 4095 - j): larger = earlier rank.  Its budget prefix is found by a
// weighted radix select over that key (8, 8, 8, 8, 8 and 4 bits, weights =
// key-group sizes): the select fixes, digit by digit, the key of the first
// rank whose group no longer fits under E; the query votes for every key
// above it (for the top key alone if even that one does not fit, for all if
// every group fits).  Keys are distinct, so the prefix is exact.
template <int KPL>
__global__ void __launch_bounds__(kPqVoteThreads) pq_votes_kernel(PqArgs a) {
  extern __shared__ uint8_t pq_sm[];
  const int M = a.d / kPqSub, Ck = a.Ck;
  float* T = reinterpret_cast<float*>(pq_sm);      // [M][16][16] codeword inner products
  float* cbq = T + M * kPqKc * kPqKc;              // [M][16][8] query codebook
  int* wsz = reinterpret_cast<int*>(cbq + M * kPqKc * kPqSub);  // [Ck] key-group sizes
  int* votes_s = wsz + Ck;                         // [Ck]
  int* hist = votes_s + Ck;                        // [8 warps][256]
  uint8_t* kc_s = reinterpret_cast<uint8_t*>(hist + 8 * 256);  // [Ck][M] key-group codes
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
  const int32_t* qoff = a.q_offsets + (size_t)bh * (a.Cq + 1);
  const int qlo = qoff[i], qhi = qoff[i + 1];
  int* h = hist + warp * 256;
  const long long E = a.E;
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
#pragma unroll
    for (int m = 0; m < 16; ++m) am[m] = __shfl_sync(0xffffffffu, code, m);
    // rank keys of this lane's key groups j = lane + 32k (0: empty or absent)
    unsigned long long key[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      const int j = lane + 32 * k;
      key[k] = 0ull;
      if (j < Ck && wsz[j] > 0) {
        float s = 0.0f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < M) s = __fadd_rn(s, T[(m * kPqKc + am[m]) * kPqKc + kc_s[j * M + m]]);
        key[k] = ((unsigned long long)pq_float_order(s) << 12) | (unsigned)(4095 - j);
      }
    }
    // weighted radix select of the first rank that does not fit
    unsigned long long prefix = 0ull, mask = 0ull;
    long long above = 0;  // weight of the keys above the current range
    bool all_fit = false;
#pragma unroll 1
    for (int pass = 0; pass < 6; ++pass) {
      const int sh = pass < 5 ? 36 - 8 * pass : 0;
      const unsigned dmask = pass < 5 ? 0xFFu : 0xFu;
      for (int b = lane; b < 256; b += 32) h[b] = 0;
      __syncwarp();
#pragma unroll
      for (int k = 0; k < KPL; ++k)
        if (key[k] != 0ull && (key[k] & mask) == prefix)
          atomicAdd(&h[(unsigned)(key[k] >> sh) & dmask], wsz[lane + 32 * k]);
      __syncwarp();
      int hb[8];
      long long lane_total = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        hb[t] = h[8 * lane + t];
        lane_total += hb[t];
      }
      // weight of the bins held by higher lanes (better keys)
      long long higher = lane_total;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long v = __shfl_down_sync(0xffffffffu, higher, o);
        if (lane + o < 32) higher += v;
      }
      higher -= lane_total;
      // this lane's highest bin where the running weight from the top passes E
      int cand = -1;
      long long cand_above = 0, run = above + higher;
#pragma unroll
      for (int t = 7; t >= 0; --t) {
        const long long before = run;
        run += hb[t];
        if (cand < 0 && run > E) {
          cand = 8 * lane + t;
          cand_above = before;
        }
      }
      const int delta = __reduce_max_sync(0xffffffffu, cand);
      if (delta < 0) {
        all_fit = true;
        break;
      }
      above = __shfl_sync(0xffffffffu, cand_above, delta >> 3);
      prefix |= (unsigned long long)delta << sh;
      mask |= (unsigned long long)dmask << sh;
      __syncwarp();
    }
    // votes: keys above kappa = prefix; the top key alone when none is above
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      if (key[k] == 0ull) continue;
      if (all_fit || key[k] > prefix || (above == 0 && key[k] == prefix)) atomicAdd(&votes_s[lane + 32 * k], 1);
    }
    __syncwarp();
  }
  __syncthreads();
  int32_t* vout = a.votes + ((size_t)bh * a.Cq + i) * Ck;
  for (int j = tid; j < Ck; j += kPqVoteThreads) vout[j] = votes_s[j];
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
  const int cmax = a.Cq > a.Ck ? a.Cq : a.Ck;
  pq_codebook_kernel<<<dim3(M, 2, a.BH), kPqCbThreads, (size_t)cmax, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t sm = (size_t)M * kPqKc * kPqKc * 4 + (size_t)M * kPqKc * kPqSub * 4 + (size_t)a.Ck * 8 + 8 * 256 * 4 +
                    (size_t)a.Ck * M;
  const int kpl = (a.Ck + 31) / 32;
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (r != cudaSuccess) return r;
    kern<<<dim3(a.Cq, a.BH), kPqVoteThreads, sm, s>>>(a);
    return cudaGetLastError();
  };
  if (kpl <= 4) return go(pq_votes_kernel<4>);
  if (kpl <= 8) return go(pq_votes_kernel<8>);
  if (kpl <= 16) return go(pq_votes_kernel<16>);
  if (kpl <= 32) return go(pq_votes_kernel<32>);
  return go(pq_votes_kernel<64>);
}

}  // namespace ig
