// Attention over the selected key blocks for 64-token blocks: the persistent
// pipelined kernel with 128-row tiles made of two query blocks (bf16).
//
// "Uncertainty-gated selection for block-sparse attention", Metodologia steps
// 2-5: one block list kv_idx per query tile, sentinel-padded so that every
// dispatch has the same shape.  "RBS-Attention" (iaonda.com), method
// paragraph: sparse prefill compatible with sparse FlashAttention, i.e.
// exact softmax attention restricted to the kept blocks.
//
// A tile holds query blocks 2m (rows 0-63, half A) and 2m + 1 (rows 64-127,
// half B) of one query head, so the M = 128 tensor-core product covers both.
// Their lists are walked side by side: step b pairs the b-th listed block of
// A with the b-th of B (when one list is longer, the other half is idle in
// the remaining steps).  A step's K (and V) stage holds the two 64-key
// blocks stacked, A's in rows 0-63 and B's in rows 64-127 (an idle half gets
// a copy of the other half's block, never used), so S = Q K^T is one 128 x
// 128 product in which each half's rows use their own 64 columns; the
// softmax writes P = 0 in the other 64, and PV = P [V_A; V_B] adds to each
// half's rows exactly its own block's contribution.  Every softmax thread
// has 32 useful scores per step, so no lane idles; half of each product's
// tensor work is discarded.
//
// Apart from the tile and the stacked stages the pipeline is that of the
// 128-token kernel: one CTA per SM walks (query head, tile) items kv-head
// major, latest tiles first; a CTA-wide step counter g drives a 4-stage K/V
// ring released by the S-done and PV-done barriers; S is double-buffered in
// TMEM with P aliased into it; Q and O are double-buffered per item.  14 warps:
//   warp 0     TMA producer (Q of item t into Q[t % 2]; the two K blocks and
//              the two V blocks of step g into ring positions 2g, 2g + 1).
//   warp 1     TMEM owner and single-thread MMA issuer (the warp reads each
//              item's lists together, then lane 0 alone waits and issues for
//              the item's steps): S(0), S(1), PV(0), S(2), PV(1), ...
//   warps 2-9  softmax: two warps per TMEM lane quadrant, 32 key columns
//              each (the columns of their rows' half); the row maximum is
//              exchanged through shared memory with the partner warp at a
//              named barrier of the two (which also tells both whether either
//              has failed a bounded wait, so they leave together); the
//              running maximum moves (and O is rescaled in TMEM) only when
//              it grows by more than 2^8.
//   warps 10-13 epilogue: O / l of the tile's 128 rows -> global memory.
// Every wait is bounded (2 s); on expiry the CTA records SBSA_ERR_TIMEOUT,
// stops issuing, drains its copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "tma_map.h"

namespace sbsa {
namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kStages = 4;  // the ring release rule relies on 4 (2 blocks)
constexpr int kThreads = 448;
// The running maximum used for exp2 moves (and O is rescaled) only when the
// row maximum exceeds it by more than 2^8 (P stays below 256).
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct PS64 {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int NA_D = D / 64;  // 128-byte swizzle atoms across d (bf16)
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;                            // Q[2]
  static constexpr int OFF_KV = 2 * Q_BYTES;                 // ring[kStages]
  static constexpr int OFF_L = OFF_KV + kStages * KV_BYTES;  // row sums [item%2][half][BM]
  static constexpr int OFF_MX = OFF_L + 4 * BM * 4;          // row max [block%2][half][BM]
  static constexpr int OFF_BAR = OFF_MX + 4 * BM * 4;
  // q_full[2] q_free[2] kv_full[S] s_full[2] p_full[2] pv_done[2]
  // o_full[2] o_free[2] l_full[2] drain
  static constexpr int NBARS = 2 + 2 + kStages + 2 + 2 + 2 + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S = 0;       // S[0], S[1]: 2 x BN columns
  static constexpr int TM_O = 2 * BN;  // O[0], O[1]: 2 x D columns
  static constexpr int TM_COLS = 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, BM, BN, false, false);
  static constexpr uint32_t IDESC_O = make_idesc(1, BM, D, false, true);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(2 * BN + 2 * D <= TM_COLS, "TMEM budget");
};

struct PSParams {
  CUtensorMap tm_q;  // box: 128 rows
  CUtensorMap tm_k;  // box: 64 rows (one key block)
  CUtensorMap tm_v;
  void* o;
  const int32_t* idx;
  const int32_t* cnt;
  int hq, n, nb, nt, group, group_shared, kmax, total;  // nb key blocks, nt tiles
  float scale_log2;
  int* status;
};

// One query block's list, read by a whole warp: lane l holds entry base + l.
struct List {
  const int32_t* ptr;
  int count;  // entries, clamped to [0, kmax]
  int valid;  // entries inside [0, qb]
  int qb;     // the query block
  int r;      // next entry to examine
  int base, val;
};

struct Item {
  int m, h, g;  // tile (query blocks 2m, 2m + 1), query head, kv head
  int steps;    // max of the two lists' valid entries
  List a, b;
};

// Opens query block qb's list (qb >= nb: an empty list).  The count and the
// first 32 entries are read together; `valid` counts entries in [0, qb].
__device__ __forceinline__ void list_open(const PSParams& p, List& L, int hs, int qb, int lane) {
  L.qb = qb;
  L.r = 0;
  L.base = 0;
  if (qb >= p.nb) {
    L.ptr = p.idx;
    L.count = 0;
    L.valid = 0;
    L.val = -1;
    return;
  }
  L.ptr = p.idx + ((size_t)hs * p.nb + qb) * p.kmax;
  const int c = p.cnt[(size_t)hs * p.nb + qb];
  const int e0 = lane < p.kmax ? L.ptr[lane] : -1;
  L.count = c < 0 ? 0 : (c > p.kmax ? p.kmax : c);
  L.val = lane < L.count ? e0 : -1;
  int v = __popc(__ballot_sync(0xFFFFFFFFu, L.val >= 0 && L.val <= qb));
  for (int base = 32; base < L.count; base += 32) {
    const int x = base + lane < L.count ? L.ptr[base + lane] : -1;
    v += __popc(__ballot_sync(0xFFFFFFFFu, x >= 0 && x <= qb));
  }
  L.valid = v;
}

// The list's next entry inside [0, qb], or -1 when none is left; entries
// outside are skipped and counted in *bad.  Warp-uniform.
__device__ __forceinline__ int list_next(List& L, int lane, int* bad) {
  while (L.r < L.count) {
    const int r = L.r++;
    const int base = r & ~31;
    if (base != L.base) {
      L.base = base;
      L.val = base + lane < L.count ? L.ptr[base + lane] : -1;
    }
    const int j = __shfl_sync(0xFFFFFFFFu, L.val, r & 31);
    if (j >= 0 && j <= L.qb) return j;
    ++*bad;
  }
  return -1;
}

// Item number t of this CTA (static round robin), kv-head major (so that a
// kv head's K and V stay in L2 while its items run), latest tiles first,
// the query heads of a group alternating.  Every lane of the warp calls it.
__device__ __forceinline__ bool load_item(const PSParams& p, int t, Item& it, int lane) {
  const long long item = (long long)blockIdx.x + (long long)t * gridDim.x;
  if (item >= p.total) return false;
  const long long per_g = (long long)p.group * p.nt;
  it.g = (int)(item / per_g);
  const int r = (int)(item % per_g);
  it.m = p.nt - 1 - r / p.group;
  it.h = it.g * p.group + r % p.group;
  const int hs = p.group_shared ? it.g : it.h;
  list_open(p, it.a, hs, 2 * it.m, lane);
  list_open(p, it.b, hs, 2 * it.m + 1, lane);
  it.steps = it.a.valid > it.b.valid ? it.a.valid : it.b.valid;
  return true;
}

__device__ __forceinline__ void record(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attend_ps64_kernel(const __grid_constant__ PSParams p) {
  using C = PS64<D>;
  constexpr int BM = C::BM, BN = C::BN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* q_free = q_full + 2;
  uint64_t* kv_full = q_free + 2;
  uint64_t* s_full = kv_full + kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 2;
  uint64_t* o_free = o_full + 2;
  uint64_t* l_full = o_free + 2;
  uint64_t* drain = l_full + 2;
  float* l_buf = reinterpret_cast<float*>(smem + C::OFF_L);
  float* mx_buf = reinterpret_cast<float*>(smem + C::OFF_MX);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sKV = smem + C::OFF_KV;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_free[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 256);
      mbar_init(&pv_done[b], 1);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], 128);
      mbar_init(&l_full[b], 256);
    }
    for (int s = 0; s < kStages; ++s) mbar_init(&kv_full[s], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    *abort_flag = 1;
    record(p.status, code);
  };
  auto wait = [&](uint64_t* b, uint32_t parity) {
    return mbar_wait_bounded(b, parity, abort_flag, kTimeoutNs);
  };

  // Producer and MMA roles run as whole warps (list entries are fetched
  // cooperatively); lane 0 issues the copies and products, and each wait's
  // outcome is broadcast so the warp leaves a loop together.
  auto warp_ok = [&](bool v) { return __shfl_sync(0xFFFFFFFFu, v, 0); };

  if (warp == 0) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    int pos = 0, t = 0, q_loaded = 0;
    bool ok = true;
    Item it;
    // Ring position q (K_b at 2b, V_b at 2b + 1) is free again once the
    // product that read it has completed: S(b) for K_b, PV(b) for V_b.  The
    // tensor core signals those completions anyway (to the softmax and for
    // rescaling), so the ring needs no release commits of its own.  With 4
    // stages, position q + 4 holds K_{b+2} or V_{b+2}, which cannot be
    // multiplied before it is loaded, so the barrier cannot run a phase
    // ahead of this wait.
    auto wait_released = [&](int q) -> bool {
      const int b = q >> 1;
      uint64_t* bar_b = (q & 1) ? &pv_done[b & 1] : &s_full[b & 1];
      return wait(bar_b, (b >> 1) & 1);
    };
    int bad = 0;
    for (; ok && load_item(p, t, it, lane); ++t) {
      const int qb = t & 1;
      bool good = true;
      if (lane == 0) {
        if (t >= 2) good = wait(&q_free[qb], ((t - 2) >> 1) & 1);
        if (good) {
          mbar_arrive_expect_tx(&q_full[qb], C::Q_BYTES);
          for (int a = 0; a < C::NA_D; ++a)
            tma_load_3d(sQ + qb * C::Q_BYTES + a * (BM * 128), &p.tm_q, &q_full[qb], a * 64,
                        it.m * BM, it.h);
        }
      }
      if (!warp_ok(good)) {
        ok = false;
        break;
      }
      q_loaded = t + 1;
      for (int b = 0; ok && b < it.steps; ++b) {
        int ja = list_next(it.a, lane, &bad);
        int jb = list_next(it.b, lane, &bad);
        // an idle half gets a copy of the other half's block
        if (ja < 0) ja = jb;
        if (jb < 0) jb = ja;
        for (int half = 0; half < 2; ++half) {
          const int st = pos % kStages;
          if (lane == 0) {
            good = pos < kStages || wait_released(pos - kStages);
            if (good) {
              mbar_arrive_expect_tx(&kv_full[st], C::KV_BYTES);
              const CUtensorMap* m = half ? &p.tm_v : &p.tm_k;
              // 64 rows of each 128-byte swizzle atom: A's block, then B's
              for (int a = 0; a < C::NA_D; ++a) {
                unsigned char* dst = sKV + st * C::KV_BYTES + a * (BN * 128);
                tma_load_3d(dst, m, &kv_full[st], a * 64, ja * 64, it.g);
                tma_load_3d(dst + 64 * 128, m, &kv_full[st], a * 64, jb * 64, it.g);
              }
            }
          }
          if (!warp_ok(good)) {
            ok = false;
            break;
          }
          ++pos;
        }
      }
    }
    if (lane == 0 && bad) record(p.status, SBSA_ERR_DEVICE);
    if (lane == 0) {
      volatile int never = 0;
      const int first = pos > kStages ? pos - kStages : 0;
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        // drain copies still landing in shared memory
        for (int u = (q_loaded >= 2 ? q_loaded - 2 : 0); u < q_loaded; ++u)
          mbar_wait_bounded(&q_full[u & 1], (u >> 1) & 1, &never, kTimeoutNs);
        for (int q = first; q < pos; ++q)
          mbar_wait_bounded(&kv_full[q % kStages], (q / kStages) & 1, &never, kTimeoutNs);
      } else {
        // wait for the MMA thread's last asynchronous releases
        for (int q = first; q < pos; ++q)
          if (!wait_released(q)) break;
        for (int u = (q_loaded >= 2 ? q_loaded - 2 : 0); u < q_loaded; ++u)
          if (!wait(&q_free[u & 1], (u >> 1) & 1)) break;
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    const uint32_t q_base = smem_u32(sQ);
    const uint32_t kv_base = smem_u32(sKV);
    // start-address-0 descriptors of the Q and K tiles (K-major, 128-byte
    // swizzle) and of V (MN-major); stage and step offsets are added to the
    // start address field
    const uint64_t q_desc0 = smem_desc(q_base, 16, 1024);
    const uint64_t k_desc0 = smem_desc(kv_base, 16, 1024);
    const uint64_t v_desc0 = smem_desc(kv_base, BN * 128, 1024);
    struct Pending {
      int g, t, b, last;  // block counter, item, block within item, last of item
    };
    Pending prev{0, 0, 0, 0};
    bool have_prev = false, ok = true;
    // lane 0 only
    auto issue_pv = [&](const Pending& pv) -> bool {
      if (!wait(&p_full[pv.g & 1], (pv.g >> 1) & 1)) return false;
      if (pv.b == 0 && pv.t >= 2 && !wait(&o_free[pv.t & 1], ((pv.t - 2) >> 1) & 1))
        return false;
      const int vpos = 2 * pv.g + 1;
      const int st = vpos % kStages;
      if (!wait(&kv_full[st], (vpos / kStages) & 1)) return false;
      tc_fence_after();
      // descriptors of the 8 K-steps differ only in the start address
      // field (16 rows of 128 bytes = 128 in units of 16 bytes per step)
      const uint64_t bd0 = v_desc0 + (uint64_t)(st * (C::KV_BYTES >> 4));
      const uint32_t a_col = tmem + C::TM_S + (pv.g & 1) * BN;
      const uint32_t o_col = tmem + C::TM_O + (pv.t & 1) * D;
      const uint32_t acc0 = pv.b > 0 ? 1u : 0u;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk)
        umma_f16_ts(o_col, a_col + kk * 8, bd0 + (uint64_t)(kk * 128), C::IDESC_O, kk > 0 ? 1u : acc0);
      umma_commit(&pv_done[pv.g & 1]);
      if (pv.last) umma_commit(&o_full[pv.t & 1]);
      return true;
    };
    int g = 0, t = 0;
    Item it;
    for (; ok && load_item(p, t, it, lane); ++t) {
      const int qb = t & 1;
      bool good = true;
      // The warp reads the item's lists together (load_item); lane 0 alone
      // waits and issues for the item's steps, and the outcome reaches the
      // warp once per item.
      if (lane == 0) {
        good = wait(&q_full[qb], (t >> 1) & 1);
        if (good) {
          tc_fence_after();
          if (it.steps == 0) {
            // nothing to multiply: release Q; the epilogue writes zeros
            umma_commit(&q_free[qb]);
            umma_commit(&o_full[qb]);
          }
        }
        for (int b = 0; good && b < it.steps; ++b) {
          const bool last = (b == it.steps - 1);
          const int kpos = 2 * g;
          const int st = kpos % kStages;
          good = wait(&kv_full[st], (kpos / kStages) & 1);
          if (good) {
            tc_fence_after();
            const uint64_t ad0 = q_desc0 + (uint64_t)(qb * (C::Q_BYTES >> 4));
            const uint64_t bd0 = k_desc0 + (uint64_t)(st * (C::KV_BYTES >> 4));
            const uint32_t s_col = tmem + C::TM_S + (g & 1) * BN;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // 32 bytes per K-step inside a 128-byte swizzle atom, then the
              // next atom (BM or BN rows of 128 bytes) every 4 steps
              const int kb = kk * 32;
              const uint64_t da = (uint64_t)(((kb / 128) * (BM * 128) + (kb % 128)) >> 4);
              const uint64_t db = (uint64_t)(((kb / 128) * (BN * 128) + (kb % 128)) >> 4);
              umma_f16_ss(s_col, ad0 + da, bd0 + db, C::IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[g & 1]);
            if (last) umma_commit(&q_free[qb]);
            if (have_prev) good = issue_pv(prev);
          }
          prev = Pending{g, t, b, last ? 1 : 0};
          have_prev = true;
          ++g;
        }
      }
      if (!warp_ok(good)) {
        ok = false;
        break;
      }
    }
    if (lane == 0) {
      if (ok && have_prev) ok = issue_pv(prev);
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait_bounded(drain, 0, &never, kTimeoutNs);
      }
    }
  } else if (warp < 10) {
    // ================================================================ softmax
    const int qd = warp & 3;             // TMEM lane quadrant
    const int hf = (warp - 2) >> 2;      // which 32 of the half's 64 key columns (and D/2 O columns)
    const int row = qd * 32 + lane;
    const int half = qd >> 1;            // 0: query block 2m (rows 0-63), 1: block 2m + 1
    const int rl = row - half * 64;      // row within its query block
    const int c0 = half * 64 + hf * 32;  // this warp's S columns
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    int g = 0, bad = 0;
    bool ok = true;
    Item it;
    for (int t = 0; ok && load_item(p, t, it, lane); ++t) {
      float m_run = -INFINITY, l_run = 0.f;
      const uint32_t o_col = tmem + lane_base + C::TM_O + (t & 1) * D + hf * (D / 2);
      int b = 0;  // steps in which this half had a block
      for (int step = 0; step < it.steps; ++step) {
        const int ja = list_next(it.a, lane, &bad);
        const int jb = list_next(it.b, lane, &bad);
        const int jh = half ? jb : ja;
        // columns c <= lim of this warp are valid keys: none when the half is
        // idle, the causal triangle on its diagonal block
        const int lim = jh < 0 ? -1 : (jh == 2 * it.m + half ? rl - hf * 32 : 31);
        const uint32_t s_col = tmem + lane_base + C::TM_S + (g & 1) * BN;
        const bool s_ok = __all_sync(0xFFFFFFFFu, wait(&s_full[g & 1], (g >> 1) & 1));
        tc_fence_after();
        float a[32];
        tmem_ld32(s_col + c0, a);
        tmem_wait_ld();
        const bool active = jh >= 0;  // uniform across the warp (one half)
        if (active && lim < 31) {
          // the diagonal block: keys past lim score -inf, so neither the
          // maximum nor the exponentials need a test (exp2(-inf) = +0)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c > lim) a[c] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) mx = fmaxf(mx, a[c]);
        // exchange the half-row maxima with the partner warp; both warps have
        // finished reading S, so P may then overwrite the first S columns
        float* mxb = mx_buf + (g & 1) * 2 * BM;
        mxb[hf * BM + row] = mx;
        // the two warps of the quadrant meet once per step; the barrier also
        // tells both whether either missed its S, so they leave together
        if (bar_red_or(1 + qd, 64, !s_ok)) {
          ok = false;
          break;
        }
        if (active) {
          mx = fmaxf(mx, mxb[(hf ^ 1) * BM + row]);
          const float m_new = fmaxf(m_run, mx * p.scale_log2);
          if (b == 0) {
            m_run = m_new;
          } else if (__any_sync(0xFFFFFFFFu, m_new > m_run + kRescaleLog2)) {
            // O must hold PV(g - 1) before it is rescaled (both warps of the
            // quadrant take this branch: they hold the same row maxima)
            const bool v_ok =
                __all_sync(0xFFFFFFFFu, wait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1));
            if (bar_red_or(1 + qd, 64, !v_ok)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float alpha = ex2_approx(m_run - m_new);
            l_run *= alpha;
            m_run = m_new;
#pragma unroll
            for (int oc = 0; oc < D / 2; oc += 16) {
              float o[16];
              tmem_ld16(o_col + oc, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) o[c] *= alpha;
              tmem_st16(o_col + oc, o);
            }
          }
        }
        // P = exp2(S * scale - m) as bf16 over this warp's 32 keys -> columns
        // [c0/2, c0/2 + 16), zeros when the half is idle (its running maximum
        // may still be -inf); zeros over 16 columns of the other half's keys
        float lsum = 0.f;
        uint32_t pk[16], zero[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) zero[c] = 0u;
        if (active) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = ex2_approx(fmaf(a[c], p.scale_log2, -m_run));
            const float p1 = ex2_approx(fmaf(a[c + 1], p.scale_log2, -m_run));
            lsum += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = 0u;
        }
        tmem_st16u(s_col + (c0 >> 1), pk);
        tmem_st16u(s_col + (1 - half) * 32 + hf * 16, zero);
        if (active) {
          l_run += lsum;
          ++b;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[g & 1]);
        ++g;
      }
      if (!ok) break;
      // hand the partial row sum to the epilogue once it is done with item t - 2
      const bool f_ok = __all_sync(0xFFFFFFFFu, t < 2 || wait(&o_free[t & 1], ((t - 2) >> 1) & 1));
      if (bar_red_or(1 + qd, 64, !f_ok)) {
        ok = false;
        break;
      }
      l_buf[((t & 1) * 2 + hf) * BM + row] = (b > 0) ? l_run : 0.f;
      mbar_arrive(&l_full[t & 1]);
    }
    if (!ok && lane == 0 && !*abort_flag) fail(SBSA_ERR_TIMEOUT);
  } else {
    // ================================================================ epilogue
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    bool ok = true;
    Item it;
    for (int t = 0; ok && load_item(p, t, it, lane); ++t) {
      if (!wait(&l_full[t & 1], (t >> 1) & 1)) ok = false;
      if (ok && !wait(&o_full[t & 1], (t >> 1) & 1)) ok = false;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float l = l_buf[((t & 1) * 2 + 0) * BM + row] + l_buf[((t & 1) * 2 + 1) * BM + row];
      const float inv_l = (it.steps > 0 && l > 0.f) ? 1.f / l : 0.f;
      const int tok = it.m * BM + row;
      const bool store = tok < p.n;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)it.h * p.n + tok) * D;
      const uint32_t o_col = tmem + lane_base + C::TM_O + (t & 1) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        if (it.steps > 0) {
          tmem_ld32(o_col + c0, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0.f;
        }
        if (store) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 v;
            v.x = pack_bf16x2(o[c + 0] * inv_l, o[c + 1] * inv_l);
            v.y = pack_bf16x2(o[c + 2] * inv_l, o[c + 3] * inv_l);
            v.z = pack_bf16x2(o[c + 4] * inv_l, o[c + 5] * inv_l);
            v.w = pack_bf16x2(o[c + 6] * inv_l, o[c + 7] * inv_l);
            *reinterpret_cast<uint4*>(orow + c0 + c) = v;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&o_free[t & 1]);
    }
    if (!ok && lane == 0 && !*abort_flag) fail(SBSA_ERR_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

template <int D>
int launch_d(const AttendArgs& a, cudaStream_t stream) {
  using C = PS64<D>;
  PSParams p{};
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&p.tm_q, dt, 2, a.q, a.hq, a.n, D, 128) ||
      !make_map(&p.tm_k, dt, 2, a.k, a.hkv, a.n, D, 64) ||
      !make_map(&p.tm_v, dt, 2, a.v, a.hkv, a.n, D, 64))
    return SBSA_ERR_CUDA;
  p.o = a.o;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.hq = a.hq;
  p.n = a.n;
  p.nb = (a.n + 63) / 64;
  p.nt = (p.nb + 1) / 2;
  p.group = a.hq / a.hkv;
  p.group_shared = a.group_shared;
  p.kmax = a.kmax;
  p.total = a.hq * p.nt;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.status = a.status;
  auto kern = attend_ps64_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SBSA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return SBSA_ERR_CUDA;
  const int grid = p.total < sms ? p.total : sms;
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SBSA_OK : SBSA_ERR_CUDA;
}

}  // namespace

int launch_attend_persistent64(const AttendArgs& a, cudaStream_t stream) {
  if (a.dtype != SBSA_BF16 || a.block != 64) return SBSA_ERR_UNSUPPORTED;
  if (a.d == 128) return launch_d<128>(a, stream);
  if (a.d == 64) return launch_d<64>(a, stream);
  return SBSA_ERR_UNSUPPORTED;
}

}  // namespace sbsa
