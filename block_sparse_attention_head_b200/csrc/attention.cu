// Sparse attention over the exact key groups plus the group-shared weighted
// sample, in one online-softmax pass (InstaGen, thelatestinai.com paper page,
// Figure 3 (d): "queries in a group share the same keys, so attention runs
// over dense blocks in one kernel"; ICLR listing abstract: the sample is
// "computed together with the top-k blocks in a single attention kernel, with
// sampled scores reweighted to account for the full skipped region").
//
// CTA = one tile of 128 queries of one query group (rows gathered from Q via
// the query permutation).  The group's key list is its exact groups (in rank
// order, contiguous ranges of the permuted K/V) followed by its m sample slots
// (gathered rows, with log-weight); it is walked in tiles of 128 keys:
//   S = Q K^T          tcgen05 (M=128, N=128, K=d), fp32 in TMEM (2 buffers)
//   P = 2^(S*scale*log2e + bias*log2e - m_run)   softmax warps, fp16 -> smem
//   O += P V           tcgen05 (M=128, N=d, K=128), fp16 operands, fp32 in TMEM
// P and V are fp16 (V converted by the gather): P <= 256 keeps 11 mantissa
// bits instead of bf16's 8, which keeps the output within 2e-3 mean relative
// error of exact arithmetic once it is rounded to bf16.
// The running max is only raised when it grows by more than 8 (log2 units), so
// P <= 256 and the O rescale (a TMEM read-modify-write) is rare.
//
// Warps: 0-1 producer (cp.async 16-byte row gathers, 128-byte swizzle; two
// rows per thread), 2 MMA issuer + TMEM owner, 3 idle, 4-7 softmax (thread =
// query row = TMEM lane).  Eight warps leave every thread 255 registers.
#include "internal.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace ig {

namespace {
constexpr int kAttnThreads = 256;
constexpr int kProducers = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct AttnSmem {
  static constexpr int kTileBytes = D * 256;  // 128 rows x D bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;          // 2 stages
  static constexpr int kV = kK + 2 * kTileBytes;      // 2 stages
  static constexpr int kP = kV + 2 * kTileBytes;      // 128 x 128 bf16
  static constexpr int kBias = kP + 32768;            // 4 warps x 2 buffers x 128 fp32
  static constexpr int kGStart = kBias + 4096;        // exact group start slots
  static constexpr int kGPre = kGStart + kAttnMaxExactGroups * 4;  // exclusive prefix of sizes
  static constexpr int kBars = kGPre + (kAttnMaxExactGroups + 1) * 4 + 12;  // 8-B aligned below
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = ((kBars + 7) & ~7) + kNumBars * 8;
  static constexpr int kBytes = kMisc + 64;
  static size_t bytes() { return 1024 + kBytes; }
};

template <typename T>
__device__ __forceinline__ const T* row_ptr(const T* base, int bh, int N, int row, int D) {
  return base + ((size_t)bh * N + row) * D;
}
}  // namespace

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1) attention_kernel(AttnArgs a) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + L::kBias);
  int* gstart = reinterpret_cast<int*>(smem + L::kGStart);
  int* gpre = reinterpret_cast<int*>(smem + L::kGPre);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ((L::kBars + 7) & ~7));
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* s_free = bars + 11;  // [2]
  uint64_t* p_full = bars + 13;
  uint64_t* pv_done = bars + 14;
  uint64_t* fin = bars + 15;
  int* misc = reinterpret_cast<int*>(smem + L::kMisc);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + 0);
  volatile int* abort_flag = misc + 1;
  int* work = misc + 2;  // group, local tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, t_glob = blockIdx.x;
  const int N = a.N, Cq = a.Cq, Ck = a.Ck;

  // ---- which (query group, tile) this CTA owns: prefix of ceil(n_i/128)
  if (warp == 0) {
    const int32_t* qoff = a.q_offsets + (size_t)bh * (Cq + 1);
    int run = 0, found_g = -1, found_t = 0;
    for (int c0 = 0; c0 < Cq && found_g < 0; c0 += 32) {
      const int c = c0 + lane;
      const int nt = (c < Cq) ? (qoff[c + 1] - qoff[c] + 127) / 128 : 0;
      int incl = nt;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = run + incl - nt;
      const bool mine = nt > 0 && t_glob >= excl && t_glob < excl + nt;
      const unsigned hit = __ballot_sync(0xffffffffu, mine);
      if (hit) {
        const int src = __ffs(hit) - 1;
        found_g = __shfl_sync(0xffffffffu, c, src);
        found_t = __shfl_sync(0xffffffffu, t_glob - excl, src);
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      work[0] = found_g;
      work[1] = found_t;
    }
  }
  __syncthreads();
  const int gi = work[0];
  if (gi < 0) return;  // tile index beyond this head's tiles
  const int lt = work[1];
  const size_t grp = (size_t)bh * Cq + gi;
  const int qlo = a.q_offsets[(size_t)bh * (Cq + 1) + gi];
  const int qhi = a.q_offsets[(size_t)bh * (Cq + 1) + gi + 1];
  const int q0 = qlo + lt * 128;
  const int nrows = min(128, qhi - q0);
  const int n_exact = a.counts[grp * 3 + 0];
  const int ns = a.counts[grp * 3 + 2];
  if (qlo < 0 || qhi > N || nrows < 1 || n_exact < 1 || n_exact > Ck || n_exact > kAttnMaxExactGroups || ns < 0 ||
      ns > a.m) {
    if (tid == 0) raise_error(kErrIndex);
    return;
  }

  // ---- exact group table: start slot and exclusive prefix of sizes
  if (warp == 0) {
    const int32_t* eg = a.exact_groups + grp * Ck;
    const int32_t* koff = a.k_offsets + (size_t)bh * (Ck + 1);
    int run = 0;
    for (int e0 = 0; e0 < n_exact; e0 += 32) {
      const int e = e0 + lane;
      int sz = 0, st = 0;
      if (e < n_exact) {
        const int g = eg[e];
        if (g >= 0 && g < Ck) {
          st = koff[g];
          sz = koff[g + 1] - st;
        } else {
          raise_error(kErrIndex);
        }
      }
      int incl = sz;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < n_exact) {
        gstart[e] = st;
        gpre[e] = run + incl - sz;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) gpre[n_exact] = run;
  }
  if (tid == 0) {
    mbar_init(q_full, kProducers);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], kProducers);
      mbar_init(&v_full[s], kProducers);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int Xi = gpre[n_exact];             // exact keys
  const int Lk = Xi + ns;                    // keys in the list
  const int ntk = (Lk + 127) / 128;          // key tiles (>= 1)
  const uint32_t q_s = smem_u32(smem + L::kQ);
  const uint32_t k_s = smem_u32(smem + L::kK);
  const uint32_t v_s = smem_u32(smem + L::kV);
  const uint32_t p_s = smem_u32(smem + L::kP);
  const int32_t* spos = a.sample_pos + grp * (size_t)a.m;
  const float* sbias = a.sample_bias + grp * (size_t)a.m;

  if (ntk < 1) {
    if (tid == 0) raise_error(kErrIndex);  // empty key list: nothing to attend
  } else if (warp < 2) {
    // ================================================================ producer
    // thread t handles tile rows t and t + 64
    for (int h = 0; h < 2; ++h) {
      const int r = tid + h * kProducers;
      bool valid = r < nrows;
      int tok = 0;
      if (valid) {
        tok = a.q_perm[(size_t)bh * N + q0 + r];
        if (tok < 0 || tok >= N) {
          raise_error(kErrIndex);
          valid = false;
          tok = 0;
        }
      }
      const __nv_bfloat16* src = row_ptr(a.Q, bh, N, tok, D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        cp_async_16(q_s + (c >> 3) * 16384 + sw128_offset(r, c & 7), src + c * 8, valid ? 16u : 0u);
    }
    cp_async_commit();
    bool ok = true;
    for (int kt = 0; kt < ntk && ok; ++kt) {
      const int s = kt & 1, use = kt >> 1;
      int pos[2];
      bool valid[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int l = kt * 128 + tid + h * kProducers;  // key slot of this row in the list
        int p = -1;
        if (l < Xi) {
          int lo = 0, hi = n_exact - 1;  // last e with gpre[e] <= l
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (gpre[mid] <= l)
              lo = mid;
            else
              hi = mid - 1;
          }
          p = gstart[lo] + (l - gpre[lo]);
        } else if (l < Lk) {
          p = spos[l - Xi];
        }
        bool v = l < Lk;
        if (v && (p < 0 || p >= N)) {
          raise_error(kErrIndex);
          v = false;
        }
        pos[h] = v ? p : 0;
        valid[h] = v;
      }
      if (kt >= 2 && !mbar_wait(&k_empty[s], (use - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t kdst = k_s + s * L::kTileBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = tid + h * kProducers;
        const __nv_bfloat16* ksrc = row_ptr(a.Kp, bh, N, pos[h], D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          cp_async_16(kdst + (c >> 3) * 16384 + sw128_offset(r, c & 7), ksrc + c * 8, valid[h] ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait<1>();  // the previous group (Q or V of the last tile) has landed
      fence_proxy_async_smem();
      mbar_arrive(kt == 0 ? q_full : &v_full[(kt - 1) & 1]);
      if (kt >= 2 && !mbar_wait(&v_empty[s], (use - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t vdst = v_s + s * L::kTileBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = tid + h * kProducers;
        const __half* vsrc = row_ptr(a.Vp, bh, N, pos[h], D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          cp_async_16(vdst + (c >> 3) * 16384 + sw128_offset(r, c & 7), vsrc + c * 8, valid[h] ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait<1>();  // this tile's K has landed
      fence_proxy_async_smem();
      mbar_arrive(&k_full[s]);
    }
    cp_async_wait<0>();
    if (ok) {
      fence_proxy_async_smem();
      mbar_arrive(&v_full[(ntk - 1) & 1]);
    }
  } else if (warp >= 4) {
    // ================================================================= softmax
    const int r = tid - 128;  // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)((r & ~31) << 16);
    float m_run = -__int_as_float(0x7f800000);
    float l_run = 0.f;
    bool ok = true;
    for (int kt = 0; kt < ntk; ++kt) {
      const int sb = kt & 1;
      // this warp's private copy of the tile's column log-weights (log2 units);
      // warp-local so an aborting thread can never strand the others
      float* wb = bias_s + ((warp - 4) * 2 + sb) * 128;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int l = kt * 128 + lane * 4 + e;
        float b;
        if (l < Xi)
          b = 0.f;
        else if (l < Lk)
          b = sbias[l - Xi] * kLog2e;
        else
          b = -__int_as_float(0x7f800000);
        wb[lane * 4 + e] = b;
      }
      __syncwarp();
      if (!mbar_wait_warp(&s_full[sb], (kt >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tmem + lane_off + sb * 128 + c4 * 32, x + c4 * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[sb]);
      const float4* bsv = reinterpret_cast<const float4*>(wb);
      float mx = -__int_as_float(0x7f800000);
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        const float4 b4 = bsv[c >> 2];
        x[c + 0] = fmaf(x[c + 0], a.scale_log2, b4.x);
        x[c + 1] = fmaf(x[c + 1], a.scale_log2, b4.y);
        x[c + 2] = fmaf(x[c + 2], a.scale_log2, b4.z);
        x[c + 3] = fmaf(x[c + 3], a.scale_log2, b4.w);
        mx = fmaxf(mx, fmaxf(fmaxf(x[c], x[c + 1]), fmaxf(x[c + 2], x[c + 3])));
      }
      const float m_new = fmaxf(m_run, mx);
      const bool rescale = m_new > m_run + kRescaleThreshold;
      float alpha = 1.f;
      if (rescale) {
        alpha = ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        x[c] = ex2_approx(x[c] - m_run);
        rs += x[c];
      }
      l_run = l_run * alpha + rs;
      if (kt >= 1) {
        if (!mbar_wait_warp(pv_done, (kt - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // tcgen05.ld/st are warp-collective: the warp rescales if any of its
        // rows needs it (alpha is 1 for the others)
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            float o[32];
            const uint32_t oaddr = tmem + lane_off + 256 + c4 * 32;
            tmem_ld32(oaddr, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(oaddr, o);
          }
          tmem_wait_st();
        }
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t addr = p_s + (c >> 3) * 16384 + sw128_offset(r, c & 7);
        st_shared_v4(addr, pack_f16x2(x[8 * c + 0], x[8 * c + 1]), pack_f16x2(x[8 * c + 2], x[8 * c + 3]),
                     pack_f16x2(x[8 * c + 4], x[8 * c + 5]), pack_f16x2(x[8 * c + 6], x[8 * c + 7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && mbar_wait_warp(pv_done, (ntk - 1) & 1, abort_flag)) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      bool valid = r < nrows;
      int tok = 0;
      if (valid) {
        tok = a.q_perm[(size_t)bh * N + q0 + r];
        if (tok < 0 || tok >= N) valid = false;
      }
      __nv_bfloat16* dst = a.O + ((size_t)bh * N + tok) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float o[32];
        tmem_ld32(tmem + lane_off + 256 + c4 * 32, o);
        tmem_wait_ld();
        if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c4 * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            d4[q] = make_uint4(pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv),
                               pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                               pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                               pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          }
        }
      }
    }
  } else if (warp == 2 && lane == 0) {
    // ===================================================================== MMA
    const uint32_t idesc_qk = umma_idesc_bf16(128, 128, false, false);
    const uint32_t idesc_pv = umma_idesc_f16kind(128, D, false, true, true);  // fp16 P and V
    bool ok = mbar_wait(q_full, 0, abort_flag);
    auto issue_pv = [&](int j) -> bool {
      if (!mbar_wait(p_full, j & 1, abort_flag)) return false;
      if (!mbar_wait(&v_full[j & 1], (j >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t vb = v_s + (j & 1) * L::kTileBytes;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint64_t ad = umma_desc_sw128(p_s + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
        const uint64_t bd = umma_desc_sw128(vb + k * 2048, 16384, 1024);
        umma_bf16_ss(tmem + 256, ad, bd, idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
      }
      umma_commit(&v_empty[j & 1]);
      umma_commit(pv_done);
      return true;
    };
    for (int kt = 0; kt < ntk && ok; ++kt) {
      const int s = kt & 1, use = kt >> 1;
      if (!mbar_wait(&k_full[s], use & 1, abort_flag)) {
        ok = false;
        break;
      }
      if (kt >= 2 && !mbar_wait(&s_free[s], (use - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t kb = k_s + s * L::kTileBytes;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t ad = umma_desc_sw128(q_s + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
        const uint64_t bd = umma_desc_sw128(kb + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
        umma_bf16_ss(tmem + s * 128, ad, bd, idesc_qk, k > 0 ? 1u : 0u);
      }
      umma_commit(&k_empty[s]);
      umma_commit(&s_full[s]);
      if (kt >= 1 && !issue_pv(kt - 1)) ok = false;
    }
    if (ok) issue_pv(ntk - 1);
    umma_commit(fin);
    mbar_wait_drain(fin, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  // tiles per head <= ceil(N/128) + Cq (each group adds at most one ragged tile)
  const long long tiles = (long long)(a.N + 127) / 128 + a.Cq;
  dim3 grid((unsigned)tiles, a.BH);
  if (a.d == 128) {
    const size_t sm = AttnSmem<128>::bytes();
    cudaError_t e =
        cudaFuncSetAttribute(attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    attention_kernel<128><<<grid, kAttnThreads, sm, s>>>(a);
  } else {
    const size_t sm = AttnSmem<64>::bytes();
    cudaError_t e =
        cudaFuncSetAttribute(attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    attention_kernel<64><<<grid, kAttnThreads, sm, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace ig
