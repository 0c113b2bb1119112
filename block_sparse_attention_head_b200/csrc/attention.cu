// Sparse attention over the exact key groups plus the group-shared weighted
// sample, in one online-softmax pass (InstaGen, thelatestinai.com paper page,
// Figure 3 (d): every query of a group attends to one common key list, so the
// work is dense tiles; ICLR listing abstract: the sampled keys run in the same
// kernel as the top-k blocks, their scores carrying a weight that stands for
// the part of the skipped region they represent).
//
// CTA = two tiles of 128 queries (Q0, Q1) of one query group, gathered from Q
// through the query permutation.  Both share the group's key list: its exact
// groups (rank order; contiguous ranges of the permuted K/V) followed by its m
// sample slots (gathered rows with log-weight w), walked in tiles of 128 keys,
// so every K/V tile brought on chip serves 256 queries.  Per key tile j and
// query tile t:
//   S_t = Q_t K_j^T + 1 w_j^T/scale    tcgen05 (M=128, N=128, bf16), fp32 in
//                          TMEM: d/16 steps over Q and K plus one side step
//                          whose 16-column operands hold (1, 1) per query row
//                          and (w_hi, w_lo) per key slot (w/scale in two bf16
//                          terms; -inf for padding slots, 0 for exact keys)
//   P_t = 2^(S_t*scale*log2e - m_t)    softmax, written back as fp16 into
//                          S_t's TMEM columns
//   O_t += P_t V_j         tcgen05 with A (P_t) read from TMEM, fp16 operands
// A CTA left with one query tile (a group's odd last tile) runs two chains
// over that tile instead: chain 0 takes the even key tiles and chain 1 the
// odd ones, each with its own S buffer, O accumulator and running max, and
// the epilogue merges the two partial softmaxes; so every CTA keeps two
// independent S -> softmax -> PV chains in flight.
// The tensor pipe alternates [PV_0(j-1), S_0(j)] and [PV_1(j-1), S_1(j)].  The
// softmax is one team of eight warps that takes the tiles in that same order
// (S_0(j), S_1(j), S_0(j+1), ...): two warps per SM sub-partition share each
// tile, one thread per half row, so one tile's exponentials run on every
// MUFU unit at once while the other tile's MMAs execute, and the two tiles'
// softmaxes never compete for the MUFU.  The two halves of a row agree on
// its running max through shared memory (one exchange per tile); each keeps
// its own partial row sum.  The running max is only raised when it grows by
// more than 8 (log2 units), so P <= 256 and the O rescale (a TMEM
// read-modify-write) is rare; it runs after S_t(j) lands, which the MMA pipe
// orders after PV_t(j-1).  P and V are fp16 (V converted by the gather): 11
// mantissa bits keep the output within 2e-3 mean relative error after its
// bf16 rounding.
//
// Warps: 0 TMEM owner and MMA warp of chain 0, 1 MMA warp of chain 1 (each
// chain's MMAs come from one elected lane, in order; two issuers keep the
// tensor pipe fed while either one waits on a barrier or sits in the issue of
// an MMA instruction, which takes about as long as the MMA itself), 2-3 and
// 12-13 producer, one warp per SM sub-partition (cp.async 16-byte
// row gathers into the 128-byte-swizzled operand layout, completion tracked
// by the stage mbarriers so the producer never blocks on memory; the key side
// rows are plain shared stores), 4-11 softmax: warp w owns TMEM lane quarter
// w mod 4 (query rows 32(w mod 4) + lane) and column half (w - 4) / 4.
#include "internal.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace ig {

namespace {
constexpr int kAttnThreads = 448;
constexpr int kProducers = 128;
constexpr int kSoftmaxThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct AttnSmem {
  static constexpr int kTileBytes = D * 256;  // 128 rows x D 16-bit
  static constexpr int kQ = 0;                          // 2 query tiles
  static constexpr int kK = kQ + 2 * kTileBytes;        // 2 stages
  static constexpr int kV = kK + 2 * kTileBytes;        // 2 stages
  // 16-column side blocks of the S product (no swizzle, 128 rows x 32 bytes):
  // ones for the query tiles, the slot log-weight over the scale for K
  static constexpr int kSideBytes = 128 * 32;
  static constexpr int kQx = kV + 2 * kTileBytes;             // shared by both query tiles
  static constexpr int kKx = kQx + kSideBytes;                // 2 stages
  static constexpr int kGStart = kKx + 2 * kSideBytes;        // exact group start slots
  static constexpr int kGPre = kGStart + kAttnMaxExactGroups * 4;  // exclusive prefix of sizes
  // half-row exchange: [2 slots][2 halves][128 rows] fp32
  static constexpr int kXch = (kGPre + (kAttnMaxExactGroups + 1) * 4 + 15) / 16 * 16;
  static constexpr int kBars = kXch + 2 * 2 * 128 * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr size_t bytes() { return 1024 + kBytes; }
};
static_assert(AttnSmem<128>::bytes() <= 232448, "shared memory budget");

template <typename T>
__device__ __forceinline__ const T* row_ptr(const T* base, int bh, int N, int row, int D) {
  return base + ((size_t)bh * N + row) * D;
}
}  // namespace

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1) attention_kernel(AttnArgs a) {
  using L = AttnSmem<D>;
  static_assert(L::kBars % 8 == 0, "barrier alignment");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* gstart = reinterpret_cast<int*>(smem + L::kGStart);
  int* gpre = reinterpret_cast<int*>(smem + L::kGPre);
  float* xch = reinterpret_cast<float*>(smem + L::kXch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2] stages
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2] query tiles
  uint64_t* p_full = bars + 11;  // [2] query tiles
  uint64_t* o_done = bars + 13;
  uint64_t* fin = bars + 14;
  int* misc = reinterpret_cast<int*>(smem + L::kMisc);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + 0);
  volatile int* abort_flag = misc + 1;
  int* work = misc + 2;  // group, local pair

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, t_glob = blockIdx.x;
  const int N = a.N, Cq = a.Cq, Ck = a.Ck;

  // ---- which (query group, pair of query tiles) this CTA owns
  if (warp == 0) {
    const int32_t* qoff = a.q_offsets + (size_t)bh * (Cq + 1);
    int run = 0, found_g = -1, found_t = 0;
    for (int c0 = 0; c0 < Cq && found_g < 0; c0 += 32) {
      const int c = c0 + lane;
      const int np = (c < Cq) ? (qoff[c + 1] - qoff[c] + 255) / 256 : 0;
      int incl = np;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = run + incl - np;
      const bool mine = np > 0 && t_glob >= excl && t_glob < excl + np;
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
  if (gi < 0) return;  // pair index beyond this head's pairs
  const int lp = work[1];
  const size_t grp = (size_t)bh * Cq + gi;
  const int qlo = a.q_offsets[(size_t)bh * (Cq + 1) + gi];
  const int qhi = a.q_offsets[(size_t)bh * (Cq + 1) + gi + 1];
  const int q0 = qlo + lp * 256;
  const int rows0 = min(128, qhi - q0);
  const int rows1 = max(0, min(128, qhi - q0 - 128));
  const int ntiles = rows1 > 0 ? 2 : 1;
  // one query tile: chains 0 and 1 split the key tiles (even / odd) of tile 0
  const bool split = ntiles == 1;
  const int n_exact = a.counts[grp * 3 + 0];
  const int ns = a.counts[grp * 3 + 2];
  if (qlo < 0 || qhi > N || rows0 < 1 || n_exact < 1 || n_exact > Ck || n_exact > kAttnMaxExactGroups || ns < 0 ||
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
  if (tid == 32) {
    // producers arrive twice per phase: their copies (cp.async) and their
    // side-block stores
    mbar_init(q_full, 2 * kProducers);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 2 * kProducers);
      mbar_init(&v_full[s], kProducers);
      // a key tile's K and V stages are freed by every chain that reads them
      mbar_init(&k_empty[s], split ? 1 : 2);
      mbar_init(&v_empty[s], split ? 1 : 2);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], kSoftmaxThreads);
    }
    mbar_init(o_done, 2);  // one commit per chain
    mbar_init(fin, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int Xi = gpre[n_exact];     // exact keys
  const int Lk = Xi + ns;           // keys in the list
  const int ntk = (Lk + 127) / 128; // key tiles
  const uint32_t q_s = smem_u32(smem + L::kQ);
  const uint32_t k_s = smem_u32(smem + L::kK);
  const uint32_t v_s = smem_u32(smem + L::kV);
  const uint32_t qx_s = smem_u32(smem + L::kQx);
  const uint32_t kx_s = smem_u32(smem + L::kKx);
  const int32_t* spos = a.sample_pos + grp * (size_t)a.m;
  const float* sbias = a.sample_bias + grp * (size_t)a.m;

  if (ntk < 1) {
    if (tid == 0) raise_error(kErrIndex);  // empty key list: nothing to attend
  } else if (warp == 2 || warp == 3 || warp >= 12) {
    // ================================================================ producer
    // four warps, one per SM sub-partition: producer warp pw owns rows
    // [32 pw, 32 pw + 32) of every K/V tile, lane l row 32 pw + l
    const int pw = warp < 4 ? warp - 2 : warp - 10;
    const int tp = 32 * pw + lane;  // 0..127
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // query rows tp and tp + 128 of the 256-row pair
      const int r = tp + 128 * h;
      const int t = h, rr = tp;
      bool valid = rr < (t == 0 ? rows0 : rows1);
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
      const uint32_t dst = q_s + t * L::kTileBytes;
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        cp_async_16(dst + (c >> 3) * 16384 + sw128_offset(rr, c & 7), src + c * 8, valid ? 16u : 0u);
    }
    cp_async_arrive_noinc(q_full);
    // Side blocks: row r of the query side is (1, 1, 0, ...), row r of a key
    // side is (w_hi, w_lo, 0, ...) with w_hi + w_lo = log-weight / scale in
    // two bf16 terms, so one more K=16 step of the S product adds the slot's
    // log-weight (and -inf for padding slots) to every score of its column.
    // Only the first 16 bytes of a key side row change per tile; this thread
    // owns row tp of every side block.
    auto side_off = [](int r, int chunk) -> uint32_t {
      return (uint32_t)((r >> 3) * 256 + chunk * 128 + (r & 7) * 16);
    };
    st_shared_v4(qx_s + side_off(tp, 0), 0x3F803F80u, 0u, 0u, 0u);  // bf16 1.0, 1.0
    st_shared_v4(qx_s + side_off(tp, 1), 0u, 0u, 0u, 0u);
    st_shared_v4(kx_s + side_off(tp, 1), 0u, 0u, 0u, 0u);
    st_shared_v4(kx_s + L::kSideBytes + side_off(tp, 1), 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    mbar_arrive(q_full);
    const float inv_scale = kLog2e / a.scale_log2;
    // slot log-weight over the scale: 0 for exact keys, -inf past the list
    auto slot_w = [&](int j) -> float {
      const int l = j * 128 + tp;
      if (l < Xi) return 0.f;
      if (l < Lk) return __ldg(sbias + (l - Xi)) * inv_scale;
      return -__int_as_float(0x7f800000);
    };
    // Slot -> permuted key position.  A lane visits increasing slots (one
    // per tile), so its exact group e (the last with gpre[e] <= slot) is
    // found by walking forward from the previous one, about one step per
    // tile, instead of a binary search per slot.
    int e = 0;
    auto key_pos = [&](int j) -> int {  // -1: padding slot
      const int l = j * 128 + tp;
      if (l < Xi) {
        while (e + 1 < n_exact && gpre[e + 1] <= l) ++e;
        return gstart[e] + (l - gpre[e]);
      }
      if (l < Lk) {
        const int p = __ldg(spos + (l - Xi));
        if (p >= N) {
          raise_error(kErrIndex);
          return -1;
        }
        return p < 0 ? -1 : p;
      }
      return -1;
    };
    constexpr int kCpr = D / 8;       // 16-byte chunks per row
    constexpr int kRpi = 32 / kCpr;   // rows per warp instruction
    constexpr int kIters = 32 / kRpi;
    const int rsub = lane / kCpr, ch = lane % kCpr;
    const uint32_t lane_dst = (uint32_t)((ch >> 3) * 16384);
    // this lane's 16-byte chunk of rows 32 pw + i*kRpi + rsub of a tile; the
    // row positions are fetched from their lanes once per tile and serve the
    // K and the V copies; one warp instruction moves whole 256-byte rows
    auto issue_rows = [&](const void* base, uint32_t dst, const int* pr) {
      // 16-byte chunks: a row is D/8 of them
      const uint4* head = reinterpret_cast<const uint4*>(base) + (size_t)bh * N * (D / 8) + ch;
#pragma unroll
      for (int i = 0; i < kIters; ++i) {
        const int r = 32 * pw + i * kRpi + rsub;
        const int p = pr[i];
        cp_async_16(dst + lane_dst + sw128_offset(r, ch & 7), head + (size_t)(p < 0 ? 0 : p) * (D / 8),
                    p < 0 ? 0u : 16u);
      }
    };
    int npos = key_pos(0);
    float nw = slot_w(0);
    for (int kt = 0; kt < ntk; ++kt) {
      const int s = kt & 1, use = kt >> 1;
      const int pos = npos;
      const float w = nw;
      if (kt + 1 < ntk) {
        npos = key_pos(kt + 1);
        nw = slot_w(kt + 1);
      }
      int pr[kIters];
#pragma unroll
      for (int i = 0; i < kIters; ++i) pr[i] = __shfl_sync(0xffffffffu, pos, i * kRpi + rsub);
      // warp-uniform waits: every lane reaches the copies together
      if (kt >= 2 && !mbar_wait_warp(&k_empty[s], (use - 1) & 1, abort_flag)) break;
      {
        const float hi = __bfloat162float(__float2bfloat16_rn(w));
        const float lo = isfinite(w) ? w - hi : 0.f;
        st_shared_v4(kx_s + s * L::kSideBytes + side_off(tp, 0), pack_bf16x2(hi, lo), 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      mbar_arrive(&k_full[s]);
      issue_rows(a.Kp, k_s + s * L::kTileBytes, pr);
      cp_async_arrive_noinc(&k_full[s]);
      if (kt >= 2 && !mbar_wait_warp(&v_empty[s], (use - 1) & 1, abort_flag)) break;
      issue_rows(a.Vp, v_s + s * L::kTileBytes, pr);
      cp_async_arrive_noinc(&v_full[s]);
    }
    cp_async_wait_all();
  } else if (warp >= 4 && warp < 12) {
    // ================================================================= softmax
    const int qd = warp & 3;               // TMEM lane quarter
    const int hf = (warp - 4) >> 2;        // column half of S and O
    const int r = 32 * qd + lane;          // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)((32 * qd) << 16);
    float m_run[2], l_run[2];
    m_run[0] = m_run[1] = -__int_as_float(0x7f800000);
    l_run[0] = l_run[1] = 0.f;
    bool ok = true;
    int xs = 0;  // exchange slot, alternating per tile visit
    for (int kt = 0; kt < ntk && ok; ++kt) {
      for (int t = 0; t < 2; ++t) {
        // chain t handles key tile kt (split: only the chain of kt's parity)
        if (split ? (kt & 1) != t : t >= ntiles) continue;
        const int ph = split ? (kt >> 1) : kt;       // visit index of chain t
        const bool first = ph == 0;                  // the chain's first key tile
        const uint32_t s_col = tmem + lane_off + (uint32_t)(128 * t + 64 * hf);
        const uint32_t o_col = tmem + lane_off + (uint32_t)(256 + 128 * t + (D / 2) * hf);
        if (!mbar_wait_warp(&s_full[t], ph & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // this thread's half row of S: 64 columns, one TMEM round trip; S
        // already carries the column log-weights (side step of the product)
        float x[64];
        tmem_ld32(s_col + 0, x);
        tmem_ld32(s_col + 32, x + 32);
        tmem_wait_ld();
        float mxp[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mxp[e] = -__int_as_float(0x7f800000);
#pragma unroll
        for (int c = 0; c < 64; c += 2) mxp[(c >> 1) & 3] = fmax3(mxp[(c >> 1) & 3], x[c], x[c + 1]);
        // The two halves of the row exchange their maxima.  Slots alternate
        // per visit: a slot is rewritten two visits later, after the partner
        // has passed the barrier of the visit in between, so after its read.
        const float hmax = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
        float* slot = xch + xs * 256;
        slot[hf * 128 + r] = hmax;
        named_bar_sync(1 + qd, 64);
        const float omax = slot[(hf ^ 1) * 128 + r];
        xs ^= 1;
        // scale after the max (scale > 0)
        const float mx = fmaxf(hmax, omax) * a.scale_log2;
        const float m_new = fmaxf(m_run[t], mx);
        const bool rescale = m_new > m_run[t] + kRescaleThreshold;
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx(m_run[t] - m_new);
          m_run[t] = m_new;
        }
        // P = 2^(x - m) as fp16 pairs: key 64hf + c -> P column 64hf + c/2, in
        // the first half of this half's own S columns (already read), packed
        // in place into slots of x already consumed
        const float neg_m = -m_run[t];
        float rsp[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t p_col = s_col;
#pragma unroll
        for (int c4 = 0; c4 < 2; ++c4) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int c = c4 * 32 + e;
            const float p0 = ex2_approx(fmaf(x[c], a.scale_log2, neg_m));
            const float p1 = ex2_approx(fmaf(x[c + 1], a.scale_log2, neg_m));
            rsp[(e >> 1) & 3] += p0 + p1;
            x[c4 * 16 + (e >> 1)] = __uint_as_float(pack_f16x2(p0, p1));
          }
          tmem_st16(p_col + c4 * 16, reinterpret_cast<const uint32_t*>(x + c4 * 16));
        }
        const float rs = (rsp[0] + rsp[1]) + (rsp[2] + rsp[3]);
        // O_t holds the chain's earlier PVs (the MMA pipe ran them before
        // S_t(kt)) and the next one waits for p_full; tcgen05.ld/st are
        // warp-collective, so the warp rescales its half of O if any of its
        // rows needs it
        if (!first && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c4 = 0; c4 < D / 64; ++c4) {
            float o[32];
            tmem_ld32(o_col + c4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(o_col + c4 * 32, o);
          }
        }
        tmem_wait_st();
        l_run[t] = l_run[t] * alpha + rs;
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
    }
    if (ok && mbar_wait_warp(o_done, 0, abort_flag)) {
      tc_fence_after();
      // row sums: the two halves' partial sums.  Every softmax thread has
      // arrived on p_full of its last tile before o_done, so each has read
      // the partner's last maximum and the whole exchange area is free.
      xch[hf * 128 + r] = l_run[0];
      xch[256 + hf * 128 + r] = l_run[1];
      named_bar_sync(1 + qd, 64);
      float lsum[2] = {l_run[0] + xch[(hf ^ 1) * 128 + r], l_run[1] + xch[256 + (hf ^ 1) * 128 + r]};
      // split: the two chains' partial softmaxes of the same rows merge with
      // weights 2^(m_c - max(m_0, m_1)); chain 1 is empty when ntk == 1
      float wgt[2] = {1.f, 1.f};
      const bool two = split && ntk > 1;
      if (two) {
        const float mm = fmaxf(m_run[0], m_run[1]);
        wgt[0] = ex2_approx(m_run[0] - mm);
        wgt[1] = ex2_approx(m_run[1] - mm);
        lsum[0] = lsum[0] * wgt[0] + lsum[1] * wgt[1];
      }
      for (int t = 0; t < ntiles; ++t) {
        const float inv = 1.f / lsum[t];
        const uint32_t o_col = tmem + lane_off + (uint32_t)(256 + 128 * t + (D / 2) * hf);
        const int nrows = t == 0 ? rows0 : rows1;
        bool valid = r < nrows;
        int tok = 0;
        if (valid) {
          tok = a.q_perm[(size_t)bh * N + q0 + 128 * t + r];
          if (tok < 0 || tok >= N) valid = false;
        }
        __nv_bfloat16* dst = a.O + ((size_t)bh * N + tok) * D + (D / 2) * hf;
#pragma unroll
        for (int c4 = 0; c4 < D / 64; ++c4) {
          float o[32];
          tmem_ld32(o_col + c4 * 32, o);
          tmem_wait_ld();
          if (two) {
            float o1[32];
            tmem_ld32(o_col + 128 + c4 * 32, o1);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = o[e] * wgt[0] + o1[e] * wgt[1];
          }
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
    }
  } else if (warp < 2) {
    // ===================================================================== MMA
    // Warp t issues chain t: S_t(j0), then for each further key tile j of the
    // chain PV_t(previous), S_t(j), and finally PV_t(last).  The whole warp
    // runs the loop and its waits in step (so descriptors and loop state are
    // warp-uniform) and one elected lane issues the MMAs and commits.
    // Descriptors are formed once and advanced by adding (byte offset >> 4)
    // to their start-address field; each wait sits right before the first
    // MMA that needs it.
    const int t = warp;
    const uint32_t idesc_qk = umma_idesc_bf16(128, 128, false, false);
    const uint32_t idesc_pv = umma_idesc_f16kind(128, D, false, true, true);  // fp16 P (TMEM) x fp16 V
    const uint64_t qd0 = umma_desc_sw128(q_s, 16, 1024);
    const uint64_t kd0 = umma_desc_sw128(k_s, 16, 1024);
    const uint64_t vd0 = umma_desc_sw128(v_s, 16384, 1024);
    const uint64_t qxd = umma_desc_noswz(qx_s, 128, 256);
    const uint64_t kxd0 = umma_desc_noswz(kx_s, 128, 256);
    constexpr uint64_t kTileStep = (uint64_t)(L::kTileBytes >> 4);
    constexpr uint64_t kSideStep = (uint64_t)(L::kSideBytes >> 4);
    const uint64_t qd = qd0 + (uint64_t)(split ? 0 : t) * kTileStep;
    const uint32_t s_t = tmem + 128 * t, o_t = tmem + 256 + 128 * t;
    // chain t's key tiles: all of them, or (split) those of parity t
    const bool active = split || t < ntiles;
    const int j0 = split ? t : 0, jstep = split ? 2 : 1;
    bool ok = mbar_wait_warp(q_full, 0, abort_flag);
    fence_proxy_async_smem();
    // O_t += P_t(j) V(j), A operand = P_t in TMEM (columns of S_t); keys
    // 16k..16k+15 of P sit in half k/4 of the tile, whose P occupies the
    // first 32 columns of that half's S columns
    auto issue_pv = [&](int j) -> bool {
      if (!mbar_wait_warp(&v_full[j & 1], (j >> 1) & 1, abort_flag)) return false;
      const int ph = split ? (j >> 1) : j;
      if (!mbar_wait_warp(&p_full[t], ph & 1, abort_flag)) return false;
      fence_proxy_async_smem();
      tc_fence_after();
      const uint64_t vd = vd0 + (uint64_t)(j & 1) * kTileStep;
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_f16_ts(o_t, s_t + 8 * k + 32 * (k >> 2), vd + (uint64_t)(k * 128), idesc_pv,
                      (ph > 0 || k > 0) ? 1u : 0u);
        umma_commit(&v_empty[j & 1]);
      }
      __syncwarp();
      return true;
    };
    auto issue_s = [&](int j) -> bool {
      if (!mbar_wait_warp(&k_full[j & 1], (j >> 1) & 1, abort_flag)) return false;
      fence_proxy_async_smem();
      tc_fence_after();
      const uint64_t kd = kd0 + (uint64_t)(j & 1) * kTileStep;
      const uint64_t kxd = kxd0 + (uint64_t)(j & 1) * kSideStep;
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t off = (uint64_t)((k >> 2) * 1024 + (k & 3) * 2);
          umma_bf16_ss(s_t, qd + off, kd + off, idesc_qk, k > 0 ? 1u : 0u);
        }
        umma_bf16_ss(s_t, qxd, kxd, idesc_qk, 1u);
        umma_commit(&s_full[t]);
        umma_commit(&k_empty[j & 1]);
      }
      __syncwarp();
      return true;
    };
    if (active) {
      int prev = -1;
      for (int j = j0; j < ntk && ok; j += jstep) {
        if (prev >= 0 && !issue_pv(prev)) {
          ok = false;
          break;
        }
        if (!issue_s(j)) {
          ok = false;
          break;
        }
        prev = j;
      }
      if (ok && prev >= 0) ok = issue_pv(prev);
    }
    if (elect_one()) {
      if (ok) umma_commit(o_done);
      umma_commit(fin);
    }
    __syncwarp();
    mbar_wait_drain(fin, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  // pairs of query tiles per head <= ceil(N/256) + Cq (one ragged pair per group)
  const long long pairs = (long long)(a.N + 255) / 256 + a.Cq;
  dim3 grid((unsigned)pairs, a.BH);
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
