// Block selection: pair scores, base branch (top-k, gated top-k or
// cumulative mass), rescue branch, union with the diagonal block, ascending
// lists with -1 padding.
//
// "Uncertainty-gated selection for block-sparse attention", technical
// summary, Metodologia: step 1 block scores from a pooling backbone, step 2
// top-k per query tile giving kv_idx, steps 3-5 a near tie at the top-k cut
// expands the tile's budget to rho*k (rho = 2) with sentinel padding so the
// dispatch shape stays uniform.  The gap form of the gate used here: fire
// when s_(k) - s_(k+1) < margin * std of the row's candidate scores.
// "RBS-Attention", method paragraph: base branch on centroid relevance and a
// rescue branch through the block radius, each with its own threshold, masks
// united.  "MiniMax presenta MSA": one selection per GQA group.
//
// Scores come from the centroids (mean backbone) or, with the K-min / K-max
// backbone ("Uncertainty-gated selection", Metodologia step 1 and
// Componibilidad: Quest-style per-coordinate upper bounds), from
// sum_d max(q_d min_d, q_d max_d) over the block's coordinate box.
//
// Layout of one CTA: R consecutive query blocks of one selection head (8
// when the scores come from a table, up to 16 when they are computed here).
// The rows' pooled queries, the kv head's radii and the table's score rows
// are staged into shared memory by bulk copies on one barrier when aligned.
// Phase 1 puts their scores against every earlier key block into shared
// memory: copied from a precomputed table (the tensor-core centroid
// scores, or the row-max tile scores), or computed here -- each thread
// streams whole key-centroid rows from L2 in 16-byte pieces and dots them
// with the R pooled queries held in shared memory (fp32 FMA; each centroid
// row is read once per CTA).  The kv head's block radii are staged beside
// them for the rescue branch.  Phase 2 gives each row to a warp: exact radix
// selection on order-preserving 32-bit keys (ties resolved by the lower
// block id), a ranked walk with 64-bit fixed-point masses for the
// cumulative-mass rule (radix selection on mass histograms past 24 blocks;
// deterministic sums), double-precision mean/std for the gate, then a ballot
// compaction that emits the ascending list.  The scans keep four 32-wide
// chunks in flight per warp.
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace sbsa {
namespace {

constexpr int kSelThreads = 256;
constexpr int kWarps = kSelThreads / 32;
constexpr int kMaxWalk = 24;  // ranked-walk steps before the radix fallback
constexpr int kShortWalk = 4;  // rank keys per lane kept for the walk
constexpr int kHistBytes = kWarps * 256 * 8;  // one 256-bin 64-bit histogram per warp
constexpr int kShortCap = 256;                // short-list keys (second half of a warp's area)
constexpr uint64_t kStageTimeoutNs = 2000000000ull;  // bound on the staging copies' wait

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Order-preserving map of a float onto uint32 (larger float -> larger key);
// -0 is folded onto +0 so equal scores give equal keys.
__device__ __forceinline__ uint32_t fkey(float f) {
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Unique descending order of the candidates: score key first, then the lower
// block id (ids are complemented so that a larger composite ranks first).
__device__ __forceinline__ uint64_t rank_key(float s, int j) {
  return ((uint64_t)fkey(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

// Key of descending rank `want` (0-based) among key(0..n).  *n_gt gets the
// number of keys strictly greater, *n_eq the number equal to it.
template <typename KeyAt>
__device__ uint32_t radix_select_keys(KeyAt key_at, int n, int want, uint32_t* hist, int* n_gt,
                                      int* n_eq) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  uint32_t rank = (uint32_t)want, above = 0, eq = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int base = 0; base < n; base += 32) {
      const int j = base + lane;
      const bool in = j < n;
      const uint32_t u = in ? key_at(j) : 0u;
      const bool match = in && ((u & pmask) == prefix);
      const uint32_t bin = (u >> shift) & 0xFFu;
      const unsigned act = __ballot_sync(0xFFFFFFFFu, match);
      if (match) {
        const unsigned peers = __match_any_sync(act, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
      }
    }
    __syncwarp();
    // lane L owns bins 255-8L ... 255-8L-7, i.e. descending order by lane
    uint32_t c[8], tot = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      c[t] = hist[255 - 8 * lane - t];
      tot += c[t];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const bool mine = excl <= rank && rank < incl;
    const int src = __ffs(__ballot_sync(0xFFFFFFFFu, mine)) - 1;
    uint32_t sel_bin = 0, sel_above = 0, sel_cnt = 0;
    if (lane == src) {
      uint32_t run = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (sel_cnt == 0 && rank < run + c[t]) {
          sel_bin = 255 - 8 * lane - t;
          sel_above = run;
          sel_cnt = c[t];
        }
        run += c[t];
      }
    }
    sel_bin = __shfl_sync(0xFFFFFFFFu, sel_bin, src);
    sel_above = __shfl_sync(0xFFFFFFFFu, sel_above, src);
    sel_cnt = __shfl_sync(0xFFFFFFFFu, sel_cnt, src);
    prefix |= sel_bin << shift;
    pmask |= 0xFFu << shift;
    rank -= sel_above;
    above += sel_above;
    eq = sel_cnt;
    __syncwarp();
  }
  *n_gt = (int)above;
  *n_eq = (int)eq;
  return prefix;
}

__device__ __forceinline__ uint32_t radix_select(const float* s, int n, int want, uint32_t* hist,
                                                 int* n_gt, int* n_eq) {
  return radix_select_keys([s](int j) { return fkey(s[j]); }, n, want, hist, n_gt, n_eq);
}

// Top-k cut through a short list.  Each lane keeps its T largest keys; the
// (need)-th largest of those 32*T values is a lower bound of the row's
// (need)-th largest key (at least `need` row keys reach it), so every key of
// rank < need is among the keys >= the bound.  Those are compacted into
// `buf` (at most `cap`) and the exact cut is taken there.  Returns false
// (nothing computed) when the short list would overflow `buf`.
template <int T>
__device__ bool topk_short(const float* s, int n, int need, uint32_t* hist, uint32_t* buf, int cap,
                           int* cnt_out) {
  const int lane = threadIdx.x & 31;
  uint32_t top[T];
#pragma unroll
  for (int q = 0; q < T; ++q) top[q] = 0u;
  for (int j = lane; j < n; j += 32) {
    uint32_t u = fkey(s[j]);
#pragma unroll
    for (int q = 0; q < T; ++q) {  // insertion into the descending list
      const uint32_t hi = max(top[q], u), lo = min(top[q], u);
      top[q] = hi;
      u = lo;
    }
  }
  // the bound: rank need-1 among the 32*T lane values (absent values are 0,
  // below every real key, and never reach rank need-1 while need <= n)
#pragma unroll
  for (int q = 0; q < T; ++q) buf[q * 32 + lane] = top[q];
  __syncwarp();
  int g, e;
  const uint32_t bound = radix_select_keys([buf](int j) { return buf[j]; }, 32 * T, need - 1,
                                           hist, &g, &e);
  __syncwarp();
  // compact the keys at or above the bound
  int m = 0;
  for (int base = 0; base < n; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < n ? fkey(s[j]) : 0u;
    const bool keep = j < n && u >= bound;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
    const int at = m + __popc(bal & ((1u << lane) - 1u));
    if (keep && at < cap) buf[at] = u;
    m += __popc(bal);
  }
  __syncwarp();
  *cnt_out = m;
  return m <= cap;
}

// Fixed-point probability of a candidate: softmax weight scaled by 2^60.
__device__ __forceinline__ uint64_t mass_weight(float s, float smax, double wscale) {
  const float e = __expf(s - smax);
  return (uint64_t)__double2ull_rn((double)e * wscale);
}

// Key v* of the candidate at which the score-ranked prefix mass first
// reaches `target` (fixed point); *w_gt = mass of the keys strictly above v*.
__device__ uint32_t radix_select_mass(const float* s, int n, float smax, double wscale,
                                      uint64_t target, unsigned long long* hist,
                                      uint64_t* w_gt) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  uint64_t above = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0ull;
    __syncwarp();
    for (int base = 0; base < n; base += 32) {
      const int j = base + lane;
      const bool in = j < n;
      const float sv = in ? s[j] : 0.f;
      const uint32_t u = in ? fkey(sv) : 0u;
      const bool match = in && ((u & pmask) == prefix);
      const uint32_t bin = (u >> shift) & 0xFFu;
      uint64_t w = match ? mass_weight(sv, smax, wscale) : 0ull;
      const unsigned act = __ballot_sync(0xFFFFFFFFu, match);
      if (match) {
        // lanes sharing a bin add their weights through one atomic
        const unsigned peers = __match_any_sync(act, bin);
        const int leader = __ffs(peers) - 1;
        unsigned rest = peers & ~(1u << leader);
        while (rest) {
          const int src = __ffs(rest) - 1;
          rest &= rest - 1;
          const uint64_t other = __shfl_sync(peers, w, src);
          if (lane == leader) w += other;
        }
        if (lane == leader && w) atomicAdd(&hist[bin], (unsigned long long)w);
      }
    }
    __syncwarp();
    uint64_t c[8], tot = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      c[t] = hist[255 - 8 * lane - t];
      tot += c[t];
    }
    uint64_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint64_t excl = incl - tot;
    const uint64_t need = target - above;  // > 0 by construction
    const bool mine = excl < need && need <= incl;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, mine);
    const int src = bal ? __ffs(bal) - 1 : 31;
    uint32_t sel_bin = 0;
    uint64_t sel_above = 0;
    if (lane == src) {
      uint64_t run = excl;
      bool done = false;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (!done && (need <= run + c[t] || (bal == 0 && t == 7))) {
          sel_bin = 255 - 8 * lane - t;
          sel_above = run;
          done = true;
        }
        if (!done) run += c[t];
      }
    }
    sel_bin = __shfl_sync(0xFFFFFFFFu, sel_bin, src);
    sel_above = __shfl_sync(0xFFFFFFFFu, sel_above, src);
    prefix |= sel_bin << shift;
    pmask |= 0xFFu << shift;
    above += sel_above;
    __syncwarp();
  }
  *w_gt = above;
  return prefix;
}

template <int DS, int R>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const __grid_constant__ SelectArgs a,
                                                            int score_stride) {
  static_assert(R <= 16, "rows per CTA");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qs = reinterpret_cast<float*>(smem_raw);                 // [R][DS]
  unsigned char* hist_base = reinterpret_cast<unsigned char*>(qs + R * DS);  // phase 2
  float* sc = reinterpret_cast<float*>(hist_base + kHistBytes);   // [R][score_stride]
  float* krs = sc + (size_t)R * score_stride;                     // [score_stride] radii (rescue)

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nrc = (a.nb + R - 1) / R;
  const int rc = nrc - 1 - (int)(blockIdx.x / a.n_sel_heads);  // longest rows first
  const int hs = (int)(blockIdx.x % a.n_sel_heads);
  const int i0 = rc * R;
  const int rows = min(R, a.nb - i0);
  const int g = hs / a.kv_div;
  const int jend = i0 + rows - 1;  // candidates needed: j < jend
  if (a.pass == 2) {
    // nothing to redo unless one of this CTA's query blocks fired
    int any = 0;
    for (int r = tid; r < rows; r += kSelThreads) any |= a.fire[i0 + r];
    if (!__syncthreads_or(any)) return;
  }

  // ---- staging: the rows' pooled queries, the kv head's radii of every
  // candidate (rescue) and, from a precomputed table, the rows' scores.  When
  // every source is 16-byte aligned, thread 0 issues them as bulk copies on
  // one barrier (one memory round trip for the whole CTA); otherwise the
  // threads copy them.
  __shared__ __align__(8) uint64_t stage_bar;
  const float* const score_base = a.scores ? a.scores + ((size_t)hs * a.nb + i0) * a.nb : nullptr;
  const bool bulk = a.qc && (reinterpret_cast<uintptr_t>(a.qc) & 15) == 0 && (a.nb & 3) == 0 &&
                    (!a.rescue || (reinterpret_cast<uintptr_t>(a.kr) & 15) == 0) &&
                    (!a.scores || (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0);
  if (bulk) {
    if (tid == 0) {
      mbar_init(&stage_bar, 1);
      fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
      // candidates rounded up to whole 16-byte pieces; nb is a multiple of 4,
      // so no row is read past its end
      const uint32_t q_bytes = (uint32_t)(rows * DS * 4);
      const uint32_t r_bytes = a.rescue ? (uint32_t)(((jend + 3) & ~3) * 4) : 0u;
      uint32_t total = q_bytes + r_bytes;
      if (score_base)
        for (int r = 0; r < rows; ++r) total += (uint32_t)(((i0 + r + 3) & ~3) * 4);
      mbar_arrive_expect_tx(&stage_bar, total);
      bulk_load(qs, a.qc + ((size_t)hs * a.nb + i0) * DS, q_bytes, &stage_bar);
      if (r_bytes) bulk_load(krs, a.kr + (size_t)g * a.nb, r_bytes, &stage_bar);
      if (score_base) {
        for (int r = 0; r < rows; ++r) {
          const uint32_t b = (uint32_t)(((i0 + r + 3) & ~3) * 4);
          if (b) bulk_load(sc + (size_t)r * score_stride, score_base + (size_t)r * a.nb, b, &stage_bar);
        }
      }
    }
    for (int e = rows * DS + tid; e < R * DS; e += kSelThreads) qs[e] = 0.f;
    volatile int never = 0;
    const bool landed = mbar_wait_bounded(&stage_bar, 0, &never, kStageTimeoutNs);
    if (__syncthreads_or(!landed)) {
      // the copies did not land in time: report it, let them finish (with a
      // bound) before the CTA's shared memory is released, and skip the rows
      if (tid == 0) record_status(a.status, SBSA_ERR_TIMEOUT);
      mbar_wait_bounded(&stage_bar, 0, &never, kStageTimeoutNs);
      return;
    }
  } else {
    for (int e = tid; e < R * DS; e += kSelThreads) {
      const int r = e / DS;
      qs[e] = (r < rows && a.qc) ? a.qc[((size_t)hs * a.nb + i0 + r) * DS + (e % DS)] : 0.f;
    }
    if (a.rescue) {
      // the kv head's radii of every candidate, read once per CTA
      const float* kr = a.kr + (size_t)g * a.nb;
      for (int j = tid; j < jend; j += kSelThreads) krs[j] = kr[j];
    }
  }
  __syncthreads();

  // ---- phase 1: scores.  Each thread owns candidate blocks j = tid + 256u
  // and streams their centroid rows (fp32) from L2 in 16-byte pieces, dotting
  // each piece with the R pooled queries read from shared memory (every lane
  // reads the same address: one broadcast per row).
  if (a.scores && !bulk) {
    // precomputed scores (centroid or row-max): copy the rows' candidates,
    // four rows' loads in flight per thread
    const float* base = score_base;
    if ((a.nb & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0) {
      for (int r0 = 0; r0 < rows; r0 += 4) {
        for (int j4 = tid; 4 * j4 < i0 + r0 + 3; j4 += kSelThreads) {
          float4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = r0 + u;
            v[u] = (r < rows && 4 * j4 < i0 + r)
                       ? __ldg(reinterpret_cast<const float4*>(base + (size_t)r * a.nb) + j4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = r0 + u;
            if (r < rows && 4 * j4 < i0 + r)
              *reinterpret_cast<float4*>(sc + r * score_stride + 4 * j4) = v[u];
          }
        }
      }
    } else {
      for (int r = 0; r < rows; ++r) {
        const float* src = base + (size_t)r * a.nb;
        for (int j = tid; j < i0 + r; j += kSelThreads) sc[r * score_stride + j] = src[j];
      }
    }
  } else if (!a.scores && a.minmax) {
    // Upper-bound backbone: s_j = sum_d max(q_d min_jd, q_d max_jd), the two
    // table rows of block j streamed like a centroid row.
    const float* km = a.kc + (size_t)g * a.nb * 2 * DS;
    for (int j = tid; j < jend; j += kSelThreads) {
      const float4* lo = reinterpret_cast<const float4*>(km + (size_t)j * 2 * DS);
      const float4* hi = lo + DS / 4;
      float acc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll 2
      for (int k4 = 0; k4 < DS / 4; ++k4) {
        const float4 l4 = __ldg(lo + k4);
        const float4 h4 = __ldg(hi + k4);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float4 q4 = *reinterpret_cast<const float4*>(qs + r * DS + 4 * k4);
          acc[r] += fmaxf(q4.x * l4.x, q4.x * h4.x);
          acc[r] += fmaxf(q4.y * l4.y, q4.y * h4.y);
          acc[r] += fmaxf(q4.z * l4.z, q4.z * h4.z);
          acc[r] += fmaxf(q4.w * l4.w, q4.w * h4.w);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) sc[r * score_stride + j] = acc[r] * a.score_scale;
    }
  }
  const float* kc = a.kc + (size_t)g * a.nb * DS;
  for (int j = (a.minmax || a.scores) ? jend : tid; j < jend; j += kSelThreads) {
    const float4* crow = reinterpret_cast<const float4*>(kc + (size_t)j * DS);
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll 4
    for (int k4 = 0; k4 < DS / 4; ++k4) {
      const float4 c4 = __ldg(crow + k4);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 q4 = *reinterpret_cast<const float4*>(qs + r * DS + 4 * k4);
        acc[r] = fmaf(q4.x, c4.x, acc[r]);
        acc[r] = fmaf(q4.y, c4.y, acc[r]);
        acc[r] = fmaf(q4.z, c4.z, acc[r]);
        acc[r] = fmaf(q4.w, c4.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) sc[r * score_stride + j] = acc[r] * a.score_scale;
  }
  __syncthreads();

  // ---- phase 2: one warp per row ----
  unsigned long long* hist64 =
      reinterpret_cast<unsigned long long*>(hist_base) + (size_t)warp * 256;
  uint32_t* hist32 = reinterpret_cast<uint32_t*>(hist64);  // 256 bins
  uint32_t* sbuf = hist32 + 256;                            // short list (kShortCap keys)
  const unsigned lt_mask = (1u << lane) - 1u;

  for (int r = warp; r < rows; r += kWarps) {
    const int i = i0 + r;
    const int n = i;  // candidates j < i
    const float* s = sc + (size_t)r * score_stride;
    int32_t* out = a.idx + ((size_t)hs * a.nb + i) * a.kmax;

    // threshold key and how many tied keys to take (in ascending id order)
    uint32_t vkey = 0xFFFFFFFFu;
    int take_eq = 0;
    bool select_all = false;
    bool walked = false;  // cumulative mass decided by the ranked walk
    uint64_t wkey = 0;    // rank key of the last block the walk kept
    uint8_t flag = 0;
    if (a.mode == SBSA_TOPK) {
      int kk = a.top_k;
      if (a.pass == 2) {
        // percentile gate, second pass: only the rows of fired tiles change
        if (!a.fire[i]) continue;
        kk = a.rho * a.top_k;
        flag |= 1;
      }
      if (n <= kk) {
        select_all = true;
        if (a.pass == 1 && lane == 0) a.sigma[(size_t)hs * a.nb + i] = __longlong_as_double(0x7FF8000000000000ll);
      } else {
        // every rank the row may need (k, k+1 for the gap test or the cut
        // margin, 2k when the gap gate fires) lies in the short list when it fits
        const int need = min(n, (a.gate ? 2 * a.top_k : kk) + 1);
        int m = 0;
        bool short_ok = false;
        if (need <= 32) short_ok = topk_short<1>(s, n, need, hist32, sbuf, kShortCap, &m);
        else if (need <= 64) short_ok = topk_short<2>(s, n, need, hist32, sbuf, kShortCap, &m);
        else if (need <= 128) short_ok = topk_short<4>(s, n, need, hist32, sbuf, kShortCap, &m);
        // keys of the row ranked by the selection: the short list or the row
        auto rank_key = [&](int want, int* gt, int* eq) {
          if (short_ok) return radix_select_keys([sbuf](int q) { return sbuf[q]; }, m, want, hist32, gt, eq);
          return radix_select(s, n, want, hist32, gt, eq);
        };
        int n_gt, n_eq;
        vkey = rank_key(kk - 1, &n_gt, &n_eq);
        take_eq = kk - n_gt;
        if (a.pass == 1) {
          // cut margin (s_(k-1) - s_(k)) / (s_(0) - s_(k)), 0-based ranks,
          // in double from the float scores; 0 when s_(0) = s_(k)
          const float last = key_float(vkey);
          float first_out = last;
          if (n_gt + n_eq < kk + 1) {
            int g1, e1;
            first_out = key_float(rank_key(kk, &g1, &e1));
          }
          int g0, e0;
          const float top = key_float(rank_key(0, &g0, &e0));
          const double sg = top == first_out
                                ? 0.0
                                : ((double)last - (double)first_out) / ((double)top - (double)first_out);
          if (lane == 0) a.sigma[(size_t)hs * a.nb + i] = sg;
        }
        if (a.gate) {
          // s_(k) and s_(k+1); population std of the candidates (double)
          const float sk = key_float(vkey);
          float sk1;
          if (n_gt + n_eq >= kk + 1) {
            sk1 = sk;
          } else {
            int g1, e1;
            sk1 = key_float(rank_key(kk, &g1, &e1));
          }
          double sum = 0.0;
          for (int j = lane; j < n; j += 32) sum += (double)s[j];
          const double mean = warp_sum_d(sum) / (double)n;
          double ss = 0.0;
          for (int j = lane; j < n; j += 32) {
            const double dlt = (double)s[j] - mean;
            ss += dlt * dlt;
          }
          const double sd = sqrt(warp_sum_d(ss) / (double)n);
          const double gap = (double)sk - (double)sk1;
          if (gap < (double)a.margin * sd) {
            flag |= 1;
            kk = 2 * a.top_k;
            if (n <= kk) {
              select_all = true;
            } else {
              vkey = rank_key(kk - 1, &n_gt, &n_eq);
              take_eq = kk - n_gt;
            }
          }
        }
      }
    } else {  // SBSA_CUMMASS
      if (n == 0) {
        select_all = true;
      } else {
        // four independent partials per lane keep four loads in flight; the
        // same pass keeps each lane's kShortWalk largest rank keys (descending)
        // for the walk below, inserting only candidates that reach the
        // lane's current smallest kept score
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        uint64_t top[kShortWalk];
#pragma unroll
        for (int q = 0; q < kShortWalk; ++q) top[q] = 0ull;
        float floor_s = -INFINITY;
        auto keep = [&](float sv, int jx) {
          if (sv >= floor_s) {
            uint64_t c = rank_key(sv, jx);
#pragma unroll
            for (int q = 0; q < kShortWalk; ++q) {
              const uint64_t hi = c > top[q] ? c : top[q];
              c = c > top[q] ? top[q] : c;
              top[q] = hi;
            }
            if (top[kShortWalk - 1]) floor_s = key_float((uint32_t)(top[kShortWalk - 1] >> 32));
          }
        };
        int j = lane;
        for (; j + 96 < n; j += 128) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float sv = s[j + 32 * u];
            m4[u] = fmaxf(m4[u], sv);
            keep(sv, j + 32 * u);
          }
        }
        for (; j < n; j += 32) {
          const float sv = s[j];
          m4[0] = fmaxf(m4[0], sv);
          keep(sv, j);
        }
        const float m = warp_max_f(fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
        double z4[4] = {0.0, 0.0, 0.0, 0.0};
        j = lane;
        for (; j + 96 < n; j += 128) {
#pragma unroll
          for (int u = 0; u < 4; ++u) z4[u] += (double)__expf(s[j + 32 * u] - m);
        }
        for (; j < n; j += 32) z4[0] += (double)__expf(s[j] - m);
        const double z = warp_sum_d((z4[0] + z4[1]) + (z4[2] + z4[3]));
        const double wscale = 1152921504606846976.0 / z;  // 2^60 / Z
        const uint64_t want = (uint64_t)ceil((double)a.mass * 1152921504606846976.0);
        // The kept prefix is usually a handful of blocks: walk the ranked
        // order one maximum at a time, accumulating fixed-point mass in the
        // same order as the definition (descending score, lower id first).
        uint64_t prev = ~0ull, cum = 0;
        int taken = 0;
        // First on the lanes' short lists: the next key of the ranked order is
        // the largest lane head, as long as no lane has used up its short list
        // while holding further candidates (whose keys it did not keep).
        {
          const int mine = lane < n ? (n - 1 - lane) / 32 + 1 : 0;  // this lane's candidates
          int used = 0;
          for (; taken < kMaxWalk && taken < n; ++taken) {
            const bool blind = used == kShortWalk && mine > kShortWalk;
            if (__any_sync(0xFFFFFFFFu, blind)) break;
            const uint64_t head = top[0];
            const uint64_t best = warp_max_u64(head);
            if (head == best) {  // keys are unique: one lane moves on
#pragma unroll
              for (int q = 0; q + 1 < kShortWalk; ++q) top[q] = top[q + 1];
              top[kShortWalk - 1] = 0ull;
              ++used;
            }
            prev = best;
            cum += mass_weight(key_float((uint32_t)(best >> 32)), m, wscale);
            if (cum >= want) {
              walked = true;
              break;
            }
          }
        }
        // then, if needed, one maximum at a time over the whole row
        for (; !walked && taken < kMaxWalk && taken < n; ++taken) {
          uint64_t b4[4] = {0, 0, 0, 0};
          int jj = lane;
          for (; jj + 96 < n; jj += 128) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint64_t c = rank_key(s[jj + 32 * u], jj + 32 * u);
              if (c < prev && c > b4[u]) b4[u] = c;
            }
          }
          for (; jj < n; jj += 32) {
            const uint64_t c = rank_key(s[jj], jj);
            if (c < prev && c > b4[0]) b4[0] = c;
          }
          const uint64_t b01 = b4[0] > b4[1] ? b4[0] : b4[1];
          const uint64_t b23 = b4[2] > b4[3] ? b4[2] : b4[3];
          const uint64_t best = warp_max_u64(b01 > b23 ? b01 : b23);
          prev = best;
          cum += mass_weight(key_float((uint32_t)(best >> 32)), m, wscale);
          if (cum >= want) {
            walked = true;
            break;
          }
        }
        if (walked) {
          wkey = prev;
        } else if (taken == n) {
          select_all = true;  // rounding kept the total below the threshold
        } else {
          // long prefix: exact radix selection on mass histograms
          uint64_t wtot = 0;
          for (int j = lane; j < n; j += 32) wtot += mass_weight(s[j], m, wscale);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) wtot += __shfl_xor_sync(0xFFFFFFFFu, wtot, o);
          uint64_t target = want > wtot ? wtot : want;
          if (target == 0) target = 1;
          if (wtot == 0) {
            select_all = true;
          } else {
            uint64_t w_gt;
            vkey = radix_select_mass(s, n, m, wscale, target, hist64, &w_gt);
            const uint64_t w_one = mass_weight(key_float(vkey), m, wscale);
            // tied keys all carry w_one; take the fewest that reach the target
            uint64_t t = w_one ? (target - w_gt + w_one - 1) / w_one : 1;
            if (t < 1) t = 1;
            if (t > (uint64_t)n) t = (uint64_t)n;
            take_eq = (int)t;
          }
        }
      }
    }

    // rescue bound scale: |q| * score_scale
    float qn_s = 0.f;
    if (a.rescue) {
      const float* qv = qs + r * DS;
      float q2 = 0.f;
      for (int c = lane; c < DS; c += 32) q2 = fmaf(qv[c], qv[c], q2);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) q2 += __shfl_xor_sync(0xFFFFFFFFu, q2, o);
      qn_s = sqrtf(q2) * a.score_scale;
    }
    // ---- compaction: ascending ids, then the diagonal, then -1 ----
    // The decisions of four 32-wide chunks are taken first (independent
    // loads), then the chunks are emitted in order.
    int written = 0, tie_seen = 0;
    bool rescued_extra = false;
    // The cut as a float: for non-NaN scores, fkey(x) > fkey(c) exactly when
    // x > c and fkey(x) == fkey(c) when x == c (-0 and +0 alike), so the
    // per-candidate tests need no keys.  A walked cut also carries its block
    // id: rank_key(x, j) >= wkey is x > c, or x == c with j <= the cut's id.
    const float cut = walked ? key_float((uint32_t)(wkey >> 32)) : key_float(vkey);
    const int cut_id = walked ? (int)(0xFFFFFFFFu - (uint32_t)wkey) : 0;
    for (int base = 0; base < n; base += 128) {
      bool bsel[4], eqk[4], resc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = base + 32 * u + lane;
        bsel[u] = false;
        eqk[u] = false;
        resc[u] = false;
        if (j < n) {
          const float sj = s[j];
          if (select_all) {
            bsel[u] = true;
          } else if (walked) {
            bsel[u] = sj > cut || (sj == cut && j <= cut_id);
          } else {
            bsel[u] = sj > cut;
            eqk[u] = sj == cut;
          }
          if (a.rescue) resc[u] = fmaf(qn_s, krs[j], sj) > a.tau;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (base + 32 * u >= n) break;  // uniform over the warp
        const unsigned eqmask = __ballot_sync(0xFFFFFFFFu, eqk[u]);
        bool basesel = bsel[u];
        if (eqk[u]) basesel = (tie_seen + __popc(eqmask & lt_mask)) < take_eq;
        tie_seen += __popc(eqmask);
        const bool sel = basesel || resc[u];
        if (resc[u] && !basesel) rescued_extra = true;
        const unsigned selmask = __ballot_sync(0xFFFFFFFFu, sel);
        const int pos = written + __popc(selmask & lt_mask);
        if (sel && pos < a.kmax - 1) out[pos] = base + 32 * u + lane;
        written += __popc(selmask);
      }
    }
    if (__any_sync(0xFFFFFFFFu, rescued_extra)) flag |= 2;
    if (written > a.kmax - 1) {
      if (lane == 0) record_status(a.status, SBSA_ERR_DEVICE);
      written = a.kmax - 1;
    }
    if (lane == 0) {
      out[written] = i;
      a.cnt[(size_t)hs * a.nb + i] = written + 1;
      if (a.flags) a.flags[(size_t)hs * a.nb + i] = flag;
    }
    // -1 padding, 16 bytes per store once the row position is aligned
    int p = written + 1;
    const int head = min(a.kmax, (p + 3) & ~3);
    if (p + lane < head) out[p + lane] = -1;
    p = head;
    if ((reinterpret_cast<uintptr_t>(out + p) & 15) == 0) {
      const int n4 = (a.kmax - p) >> 2;
      int4* o4 = reinterpret_cast<int4*>(out + p);
      for (int q = lane; q < n4; q += 32) o4[q] = make_int4(-1, -1, -1, -1);
      p += 4 * n4;
    }
    for (int q = p + lane; q < a.kmax; q += 32) out[q] = -1;
    __syncwarp();
  }
}

template <int DS, int R>
cudaError_t launch_rows(const SelectArgs& a, cudaStream_t stream) {
  const int stride = (a.nb + 3) & ~3;
  const size_t smem = (size_t)R * DS * 4 + kHistBytes + (size_t)R * stride * 4 +
                      (a.rescue ? (size_t)stride * 4 : 0);
  auto kern = select_kernel<DS, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long nrc = (a.nb + R - 1) / R;
  const long long grid = nrc * a.n_sel_heads;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, kSelThreads, smem, stream>>>(a, stride);
  return cudaGetLastError();
}

// Percentile gate, first half of the tile decisions: the sum of each query
// tile's cut margins over this call's selection heads, in head order
// (double).  Tiles with at most k candidates have no margin (NaN).
__global__ void __launch_bounds__(256) gate_sums_kernel(const double* sigma, double* sums,
                                                        int n_sel_heads, int nb) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += gridDim.x * blockDim.x) {
    double tot = 0.0;
    for (int h = 0; h < n_sel_heads; ++h) tot += sigma[(size_t)h * nb + i];
    sums[i] = tot;
  }
}

// Percentile gate, second half: the mean margin of each tile is its sum over
// all selection heads divided by their number; the floor(q T) smallest of the
// T tiles with more than k candidates fire, lower tile first on equal means.
// One CTA; the means live in shared memory.
__global__ void __launch_bounds__(1024) gate_fire_kernel(const double* sums, uint8_t* fire,
                                                         int total_heads, int nb, int top_k,
                                                         float quantile) {
  extern __shared__ double sbar[];
  for (int i = threadIdx.x; i < nb; i += blockDim.x) sbar[i] = sums[i] / (double)total_heads;
  __syncthreads();
  const int t_eligible = nb - 1 - top_k > 0 ? nb - 1 - top_k : 0;
  const int n_fire = (int)floor((double)quantile * (double)t_eligible);
  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    uint8_t f = 0;
    if (i > top_k && n_fire > 0) {
      const double si = sbar[i];
      int rank = 0;
      for (int j = top_k + 1; j < nb; ++j) {
        const double sj = sbar[j];
        rank += (sj < si || (sj == si && j < i)) ? 1 : 0;
      }
      f = rank < n_fire ? 1 : 0;
    }
    fire[i] = f;
  }
}

// Shared memory of a CTA of R score rows: the R pooled queries and score
// rows, the per-warp histograms, the kv head's radii when rescuing.
constexpr size_t kSelectBudget = 200 * 1024;
size_t select_smem(int rows, int nb, int ds, int rescue) {
  const size_t stride = (size_t)((nb + 3) & ~3) * 4;
  return kHistBytes + (rescue ? stride : 0) + (size_t)rows * (stride + (size_t)ds * 4);
}

template <int DS>
cudaError_t launch_ds(const SelectArgs& a, cudaStream_t stream) {
  // rows per CTA.  Scores read from a precomputed table: 8, so that three
  // CTAs (24 warps) fit an SM and hide the per-row latency.  Scores computed
  // here: as many (up to 16) as the score rows allow in shared memory, since
  // more rows per CTA means fewer reads of each centroid row from L2.
  if (a.scores && select_smem(8, a.nb, DS, a.rescue) <= kSelectBudget)
    return launch_rows<DS, 8>(a, stream);
  if (select_smem(16, a.nb, DS, a.rescue) <= kSelectBudget) return launch_rows<DS, 16>(a, stream);
  if (select_smem(8, a.nb, DS, a.rescue) <= kSelectBudget) return launch_rows<DS, 8>(a, stream);
  if (select_smem(4, a.nb, DS, a.rescue) <= kSelectBudget) return launch_rows<DS, 4>(a, stream);
  if (select_smem(2, a.nb, DS, a.rescue) <= kSelectBudget) return launch_rows<DS, 2>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gate_sums(const double* sigma, double* sums, int n_sel_heads, int nb,
                             cudaStream_t stream) {
  const int blocks = (nb + 255) / 256;
  gate_sums_kernel<<<blocks, 256, 0, stream>>>(sigma, sums, n_sel_heads, nb);
  return cudaGetLastError();
}

cudaError_t launch_gate_fire(const double* sums, uint8_t* fire, int total_heads, int nb,
                             int top_k, float quantile, cudaStream_t stream) {
  const size_t smem = (size_t)nb * sizeof(double);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(gate_fire_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return cudaErrorInvalidValue;
  gate_fire_kernel<<<1, 1024, smem, stream>>>(sums, fire, total_heads, nb, top_k, quantile);
  return cudaGetLastError();
}

bool select_fits(int nb, int ds, int rescue) {
  return select_smem(2, nb, ds, rescue) <= kSelectBudget;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  return a.ds == 128 ? launch_ds<128>(a, stream) : launch_ds<64>(a, stream);
}

}  // namespace sbsa
