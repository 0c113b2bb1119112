// Centroid scoring, exact set and group-shared importance sampling
// (InstaGen abstract: the highest-scoring keys are attended exactly, the rest
// are stood in for by a sample whose draw probability follows the estimated
// attention and whose scores are weighted by the inverse of that probability;
// one sample per query cluster, used by all of its queries; thelatestinai.com
// paper page, Figure 3 (b), (c)).
//
// Everything that decides an index is integer arithmetic or a correctly
// rounded fp32 operation in a fixed order (fused multiply-add chain for the
// scores, integer weights, uint64 CDF, Philox4x32-10), so the indices are
// reproducible bit for bit on any conforming implementation.
#include "internal.cuh"
#include "ptx.cuh"

namespace ig {

namespace {
constexpr int kSelThreads = 512;
constexpr unsigned long long kKeyJ = 0xFFFull;  // group index field of a rank key
constexpr int kSelMaxCk = 4096;

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC 2011): ten rounds of two
// 32x32 -> 64-bit products with the Philox multipliers, key bumped by the
// Weyl increments between rounds.
struct U4 {
  uint32_t x, y, z, w;
};
__device__ __forceinline__ U4 philox4x32_10(U4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
  }
  return c;
}

// Integer weight q in [1, 2^24] ~ 2^24 * exp(s - smax): y = (s - smax) log2(e)
// = n + f, 2^f by its degree-6 Taylor series in f ln 2 (Horner, fused
// multiply-adds), scaled by 2^(24 + n) exactly, floored.
__device__ __forceinline__ uint32_t group_weight(float s, float smax) {
  const float y = __fmul_rn(__fsub_rn(s, smax), 0x1.715476p+0f);  // log2(e) in fp32
  if (y < -24.0f) return 1u;
  const float n = floorf(y);
  const float f = __fsub_rn(y, n);
  float p = 0x1.430912p-13f;              // (ln 2)^6 / 6!
  p = __fmaf_rn(p, f, 0x1.5d87fep-10f);   // (ln 2)^5 / 5!
  p = __fmaf_rn(p, f, 0x1.3b2ab6p-7f);    // (ln 2)^4 / 4!
  p = __fmaf_rn(p, f, 0x1.c6b08ep-5f);    // (ln 2)^3 / 3!
  p = __fmaf_rn(p, f, 0x1.ebfbe0p-3f);    // (ln 2)^2 / 2!
  p = __fmaf_rn(p, f, 0x1.62e430p-1f);    // ln 2
  p = __fmaf_rn(p, f, 1.0f);
  const int e = 24 + (int)n;              // 0 .. 24
  const float scaled = __fmul_rn(p, __int_as_float((127 + e) << 23));
  const uint32_t q = (uint32_t)floorf(scaled);
  return q < 1u ? 1u : q;
}

// Order-preserving map of a float to uint32 (+0 and -0 made equal first).
__device__ __forceinline__ uint32_t float_order(float s) {
  if (s == 0.0f) s = 0.0f;
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// In-place inclusive scan of n uint64 values in shared memory.
__device__ void block_incl_scan_u64(unsigned long long* v, int n, unsigned long long* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  unsigned long long run = 0;
  for (int i = b0; i < b1; ++i) {
    run += v[i];
    v[i] = run;
  }
  unsigned long long incl = run;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < kSelThreads / 32 ? warp_tot[lane] : 0ull;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < kSelThreads / 32) warp_tot[lane] = w;
  }
  __syncthreads();
  const unsigned long long off = (incl - run) + (warp > 0 ? warp_tot[warp - 1] : 0ull);
  for (int i = b0; i < b1; ++i) v[i] += off;
  __syncthreads();
}
}  // namespace

// One CTA per (query group i, head bh).
__global__ void __launch_bounds__(kSelThreads)
    select_sample_kernel(SelectArgs a, int ck_pow2) {
  extern __shared__ uint8_t sm[];
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(sm);      // [ck_pow2]
  unsigned long long* cdf = keys + ck_pow2;                                   // [Ck]
  unsigned long long* wtot = cdf + a.Ck;                                      // [32]
  float* S = reinterpret_cast<float*>(wtot + 32);                             // [Ck]
  uint32_t* qw = reinterpret_cast<uint32_t*>(S + a.Ck);                       // [Ck]
  int* koff = reinterpret_cast<int*>(qw + a.Ck);                              // [Ck+1]
  float* lq = reinterpret_cast<float*>(koff + a.Ck + 1);                      // [Ck] logf(q_j)
  float* cqrow = lq + a.Ck;                                                   // [d]
  unsigned long long* qinv = reinterpret_cast<unsigned long long*>(
      (reinterpret_cast<uintptr_t>(cqrow + a.d) + 7) & ~uintptr_t(7));         // [Ck] floor((2^64-1)/q_j)
  __shared__ int s_nexact, s_nskipped;
  __shared__ unsigned s_smax_bits;
  __shared__ long long s_exact_keys;

  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int Ck = a.Ck, d = a.d;
  const size_t gi = (size_t)bh * a.Cq + i;

  for (int k = tid; k < d; k += kSelThreads) cqrow[k] = a.cq[gi * d + k];
  for (int j = tid; j <= Ck; j += kSelThreads) koff[j] = a.k_offsets[(size_t)bh * (Ck + 1) + j];
  if (tid == 0) {
    s_nexact = 0;
    s_nskipped = 0;
    s_smax_bits = 0u;
    s_exact_keys = 0;
  }
  __syncthreads();

  // (b) scores: fp32 fused multiply-add chain over k = 0..d-1, then * scale
  // (the row is fetched 32 values at a time with 16-byte loads, all in
  // flight together, ahead of the serial fma chain)
  for (int j = tid; j < Ck; j += kSelThreads) {
    const float4* ckr = reinterpret_cast<const float4*>(a.ck + ((size_t)bh * Ck + j) * d);
    float acc = 0.0f;
    for (int k0 = 0; k0 < d; k0 += 32) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(ckr + k0 / 4 + u);
      const float* f = reinterpret_cast<const float*>(v);
#pragma unroll
      for (int e = 0; e < 32; ++e) acc = __fmaf_rn(cqrow[k0 + e], f[e], acc);
    }
    S[j] = __fmul_rn(acc, a.scale);
  }
  __syncthreads();

  if (a.top_p) {
    // Top-p selection (the comparator of the Figure 2 caption, SVG2-style):
    // mass W_j = |K_j| q_j with the integer weights taken over every
    // non-empty group, ranked by W descending (ties: lower j; rank key =
    // (2^44 - 1 - W) << 12 | j), kept until the share of the total reaches
    // p_fix / 2^20 and the kept keys reach floor_keys; no sample.
    constexpr unsigned long long kMaxW = (1ull << 44) - 1;
    for (int j = tid; j < Ck; j += kSelThreads)
      if (koff[j + 1] > koff[j]) atomicMax(&s_smax_bits, float_order(S[j]));
    if (tid == 0) s_nexact = 0x7fffffff;  // first rank that satisfies both conditions
    __syncthreads();
    const uint32_t ob_all = s_smax_bits;
    const float smax_all = __uint_as_float((ob_all & 0x80000000u) ? (ob_all & 0x7fffffffu) : ~ob_all);
    for (int j = tid; j < ck_pow2; j += kSelThreads) {
      unsigned long long key = ~0ull;
      if (j < Ck && koff[j + 1] > koff[j]) {
        const unsigned long long W =
            (unsigned long long)(koff[j + 1] - koff[j]) * group_weight(S[j], smax_all);
        key = ((kMaxW - W) << 12) | (unsigned)j;
      }
      keys[j] = key;
    }
    __syncthreads();
    for (int k = 2; k <= ck_pow2; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        for (int x = tid; x < ck_pow2; x += kSelThreads) {
          const int y = x ^ jj;
          if (y > x) {
            const unsigned long long u = keys[x], v = keys[y];
            const bool up = (x & k) == 0;
            if ((u > v) == up) {
              keys[x] = v;
              keys[y] = u;
            }
          }
        }
        __syncthreads();
      }
    }
    // cumulative mass (cdf) and kept keys (qinv as scratch) in rank order
    for (int r = tid; r < Ck; r += kSelThreads) {
      const unsigned long long key = keys[r];
      const bool ne = key != ~0ull;
      const int j = (int)(key & kKeyJ);
      cdf[r] = ne ? kMaxW - (key >> 12) : 0ull;
      qinv[r] = ne ? (unsigned long long)(koff[j + 1] - koff[j]) : 0ull;
    }
    __syncthreads();
    block_incl_scan_u64(cdf, Ck, wtot);
    block_incl_scan_u64(qinv, Ck, wtot);
    const unsigned long long T = cdf[Ck - 1];
    int nz_local = 0;
    for (int r = tid; r < Ck; r += kSelThreads) {
      if (keys[r] == ~0ull) continue;
      ++nz_local;
      if (cdf[r] * 1048576ull >= (unsigned long long)a.p_fix * T && qinv[r] >= (unsigned long long)a.floor_keys)
        atomicMin(&s_nexact, r);
    }
    atomicAdd(&s_nskipped, nz_local);  // here: the number of non-empty groups
    __syncthreads();
    const int n_keep = s_nexact == 0x7fffffff ? s_nskipped : s_nexact + 1;
    int32_t* ex_top = a.exact_groups + gi * Ck;
    for (int r = tid; r < Ck; r += kSelThreads) ex_top[r] = r < n_keep ? (int32_t)(keys[r] & kKeyJ) : -1;
    for (long long t = tid; t < a.m; t += kSelThreads) {
      a.sample_pos[gi * a.m + t] = -1;
      a.sample_bias[gi * a.m + t] = 0.0f;
    }
    if (tid == 0) {
      a.counts[gi * 3 + 0] = n_keep;
      a.counts[gi * 3 + 1] = n_keep > 0 ? (int32_t)qinv[n_keep - 1] : 0;
      a.counts[gi * 3 + 2] = 0;
    }
    return;
  }

  // rank the non-empty groups: S descending, j ascending (bitonic sort of
  // keys; j < 4096 sits in the low 12 bits).  With votes (product-quantised
  // voting) the votes, descending, come first (20 bits, saturated).
  for (int j = tid; j < ck_pow2; j += kSelThreads) {
    unsigned long long key = ~0ull;
    if (j < Ck && koff[j + 1] > koff[j]) {
      key = ((unsigned long long)(~float_order(S[j])) << 12) | (unsigned)j;
      if (a.votes) {
        const int v = min(max(a.votes[gi * Ck + j], 0), 0xFFFFF);
        key |= (unsigned long long)(0xFFFFF - v) << 44;
      }
    }
    keys[j] = key;
  }
  __syncthreads();
  for (int k = 2; k <= ck_pow2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int x = tid; x < ck_pow2; x += kSelThreads) {
        const int y = x ^ jj;
        if (y > x) {
          const unsigned long long u = keys[x], v = keys[y];
          const bool up = (x & k) == 0;
          if ((u > v) == up) {
            keys[x] = v;
            keys[y] = u;
          }
        }
      }
      __syncthreads();
    }
  }

  // exact set: rank 0, then while the running key count stays <= E
  for (int r = tid; r < Ck; r += kSelThreads) {
    const unsigned long long key = keys[r];
    cdf[r] = (key == ~0ull) ? 0ull : (unsigned long long)(koff[(key & kKeyJ) + 1] - koff[key & kKeyJ]);
  }
  __syncthreads();
  block_incl_scan_u64(cdf, Ck, wtot);  // cdf[r] = keys in ranks 0..r
  for (int r = tid; r < Ck; r += kSelThreads) {
    const bool nonempty = keys[r] != ~0ull;
    const bool incl = nonempty && (r == 0 || cdf[r] <= (unsigned long long)a.E);
    if (incl && (r + 1 == Ck || !(keys[r + 1] != ~0ull && cdf[r + 1] <= (unsigned long long)a.E))) {
      s_nexact = r + 1;  // last included rank (the included ranks are a prefix)
      s_exact_keys = (long long)cdf[r];
    }
  }
  __syncthreads();
  const int n_exact = s_nexact;
  int32_t* ex_out = a.exact_groups + gi * Ck;
  for (int r = tid; r < Ck; r += kSelThreads) ex_out[r] = r < n_exact ? (int32_t)(keys[r] & kKeyJ) : -1;
  // qw doubles as the exact-membership flag: 0 = exact or empty, 1 = skipped (for now)
  for (int j = tid; j < Ck; j += kSelThreads) qw[j] = (koff[j + 1] > koff[j]) ? 1u : 0u;
  __syncthreads();
  for (int r = tid; r < n_exact; r += kSelThreads) qw[keys[r] & kKeyJ] = 0u;
  __syncthreads();

  // pi over the skipped groups
  for (int j = tid; j < Ck; j += kSelThreads) {
    if (qw[j]) {
      atomicAdd(&s_nskipped, 1);
      atomicMax(&s_smax_bits, float_order(S[j]));
    }
  }
  __syncthreads();
  const bool any_skipped = s_nskipped > 0;
  const uint32_t ob = s_smax_bits;
  const float smax = __uint_as_float((ob & 0x80000000u) ? (ob & 0x7fffffffu) : ~ob);
  for (int j = tid; j < Ck; j += kSelThreads) {
    uint32_t q = 0u;
    if (qw[j]) q = (a.mode == 1) ? 1u : group_weight(S[j], smax);
    qw[j] = q;
    lq[j] = logf((float)q);  // the draws' log-weights take it from here
    qinv[j] = q ? ~0ull / q : 0ull;
    cdf[j] = (unsigned long long)(koff[j + 1] - koff[j]) * q;
  }
  __syncthreads();
  block_incl_scan_u64(cdf, Ck, wtot);  // inclusive CDF over j ascending
  const unsigned long long T = cdf[Ck - 1];

  const long long m = a.m;
  const long long draws = any_skipped ? m : 0;
  const float logT = logf((float)T);
  const float logm = draws > 0 ? logf((float)draws) : 0.0f;
  const uint32_t k0 = (uint32_t)(a.seed & 0xffffffffull), k1 = (uint32_t)(a.seed >> 32);
  for (long long t = tid; t < m; t += kSelThreads) {
    int32_t pos = -1;
    float bias = 0.0f;
    if (t < draws) {
      const U4 rnd = philox4x32_10(U4{(uint32_t)t, (uint32_t)i, (uint32_t)(a.bh0 + bh), a.layer}, k0, k1);
      const unsigned long long u = ((unsigned long long)rnd.y << 32) | rnd.x;
      const unsigned long long r = __umul64hi(u, T);
      int lo = 0, hi = Ck - 1;  // first j with cdf[j] > r
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cdf[mid] > r)
          hi = mid;
        else
          lo = mid + 1;
      }
      const int j = lo;
      const uint32_t q = qw[j];
      if (q == 0u || cdf[j] <= r) {
        raise_error(kErrSampling);
      } else {
        const unsigned long long start = cdf[j] - (unsigned long long)(koff[j + 1] - koff[j]) * q;
        // floor((r - start) / q) by the group's reciprocal: with
        // qinv = floor((2^64-1)/q) and x < 2^56, mulhi(x, qinv) is the
        // quotient or one less; one remainder test makes it exact
        const unsigned long long x = r - start;
        unsigned long long o = __umul64hi(x, qinv[j]);
        if (x - o * q >= q) ++o;
        pos = koff[j] + (int32_t)o;
        bias = logT - lq[j] - logm;
      }
    }
    a.sample_pos[gi * m + t] = pos;
    a.sample_bias[gi * m + t] = bias;
  }
  if (tid == 0) {
    a.counts[gi * 3 + 0] = n_exact;
    a.counts[gi * 3 + 1] = (int32_t)s_exact_keys;
    a.counts[gi * 3 + 2] = (int32_t)draws;
  }
}

cudaError_t launch_select_sample(const SelectArgs& a, cudaStream_t s) {
  int p2 = 1;
  while (p2 < a.Ck) p2 <<= 1;
  const size_t sm = (size_t)p2 * 8 + (size_t)a.Ck * 8 + 32 * 8 + (size_t)a.Ck * 4 * 3 + (size_t)(a.Ck + 1) * 4 +
                    (size_t)a.d * 4 + 8 + (size_t)a.Ck * 8 + 16;
  cudaError_t e = cudaFuncSetAttribute(select_sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Cq, a.BH);
  select_sample_kernel<<<grid, kSelThreads, sm, s>>>(a, p2);
  return cudaGetLastError();
}

}  // namespace ig
