// Attention over the selected key blocks with two independent query tiles in
// flight per CTA (bf16, 128-token blocks, one block list per query head).
//
// "RBS-Attention" (iaonda.com), method paragraph: sparse prefill compatible
// with sparse FlashAttention, i.e. exact softmax attention restricted to the
// kept blocks.  "Uncertainty-gated selection for block-sparse attention",
// Metodologia step 2: one list kv_idx per query tile.
//
// Work: one item per (query head, query block).  Items are taken kv-head
// major -- all items reading kv head 0, then kv head 1, ... -- so that the K
// and V tiles the lists name (2 * N * d * 2 bytes per kv head) stay in L2
// while their items run; within a kv head the latest query blocks (longest
// lists) come first and the query heads of the group alternate.  One CTA per
// SM takes items blockIdx.x + t * gridDim.x; its items alternate between two
// slots (even t, odd t).  Each slot has its own Q tile in shared memory and
// its own S (P aliased into it) and O accumulators in TMEM, so one slot's
// softmax runs while the tensor core multiplies the other slot's tiles.
// 10 warps:
//   warp 0     TMA producer: the K and V tiles of both slots, in the order the
//              tensor core consumes them, through a 5-stage ring; a slot's Q
//              tile once the last S product of its previous item is done.
//   warp 1     TMEM owner and single-thread MMA issuer.  Per step, slot 0 then
//              slot 1: O_x += P_x V (the slot's previous block, once its
//              softmax has written P), then S_x = Q_x K^T (its next block).
//              The commit announcing S_x completes after the PV before it, so
//              it also releases both ring positions of the step (that V and
//              this K): one commit per block.
//   warps 2-5  softmax and epilogue of slot 0, warps 6-9 of slot 1: one query
//              row per thread, a block's 128 scores held in registers; the
//              running maximum moves (and O is rescaled in TMEM) only when the
//              row maximum exceeds it by more than 2^8; P (bf16) is written
//              over the first half of S; at the end of an item O / l goes to
//              global memory.
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
constexpr int kStages = 5;
constexpr int kThreads = 320;
// S barriers per slot, used round robin.  The producer waits on them to reuse
// a ring position; with four, the tensor core cannot complete a later phase
// of the same barrier before that wait (it would have to consume more
// positions than the ring holds beyond the awaited one).
constexpr int kSBars = 4;
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct DC {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int NA_D = D / 64;  // 128-byte swizzle atoms across d (bf16)
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;                 // Q[slot]
  static constexpr int OFF_KV = 2 * Q_BYTES;      // ring[kStages]
  static constexpr int OFF_BAR = OFF_KV + kStages * KV_BYTES;
  // kv_full[S] q_full[2] q_free[2] s_full[2][kSBars] p_full[2] o_full[2] drain
  static constexpr int NBARS = kStages + 2 + 2 + 2 * kSBars + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S = 0;       // S[slot]: BN columns each
  static constexpr int TM_O = 2 * BN;  // O[slot]: D columns each
  static constexpr int TM_COLS = 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, BM, BN, false, false);
  static constexpr uint32_t IDESC_O = make_idesc(1, BM, D, false, true);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(2 * BN + 2 * D <= TM_COLS, "TMEM budget");
};

struct DuoParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void* o;
  const int32_t* idx;
  const int32_t* cnt;
  int hq, n, nb, group, kmax;
  long long total;
  float scale_log2;
  int* status;
};

// One slot's current item, read by a whole warp: lane l holds list entry
// chunk_base + l.
struct Stream {
  int t;           // CTA-local item number
  int i, h, g;     // query block, query head, kv head
  const int32_t* list;
  int count;       // list entries (clamped to [0, kmax])
  int valid;       // entries inside [0, i]
  int r;           // next entry to examine
  int b;           // valid entries consumed
  int chunk_base, chunk_val;
  bool live;
};

// Opens CTA-local item t; every lane of the warp must call it together.
__device__ __forceinline__ bool stream_open(const DuoParams& p, Stream& s, int t, int lane) {
  s.t = t;
  const long long u = (long long)blockIdx.x + (long long)t * gridDim.x;
  s.live = u < p.total;
  if (!s.live) return false;
  // kv-head-major, latest query block first, query heads of the group alternating
  const long long per_g = (long long)p.group * p.nb;
  s.g = (int)(u / per_g);
  const int rr = (int)(u % per_g);
  s.i = p.nb - 1 - rr / p.group;
  s.h = s.g * p.group + rr % p.group;
  s.list = p.idx + ((size_t)s.h * p.nb + s.i) * p.kmax;
  // the count and the first 32 entries are read together (one round trip)
  const int c = p.cnt[(size_t)s.h * p.nb + s.i];
  const int e0 = lane < p.kmax ? s.list[lane] : -1;
  s.count = c < 0 ? 0 : (c > p.kmax ? p.kmax : c);
  s.chunk_base = 0;
  s.chunk_val = lane < s.count ? e0 : -1;
  int v = __popc(__ballot_sync(0xFFFFFFFFu, s.chunk_val >= 0 && s.chunk_val <= s.i));
  for (int base = 32; base < s.count; base += 32) {
    const int x = base + lane < s.count ? s.list[base + lane] : -1;
    v += __popc(__ballot_sync(0xFFFFFFFFu, x >= 0 && x <= s.i));
  }
  s.valid = v;
  s.r = 0;
  s.b = 0;
  return true;
}

// List entry r of the current item (uniform r across the warp).
__device__ __forceinline__ int stream_entry(Stream& s, int r, int lane) {
  const int base = r & ~31;
  if (base != s.chunk_base) {
    s.chunk_base = base;
    s.chunk_val = base + lane < s.count ? s.list[base + lane] : -1;
  }
  return __shfl_sync(0xFFFFFFFFu, s.chunk_val, r & 31);
}

// The slot's next valid block, moving on to the slot's next item (t + 2)
// when the current one is exhausted; items without valid entries are passed
// over (their softmax warps write zeros).  Entries outside [0, i] are
// skipped and counted in *bad.
__device__ __forceinline__ bool stream_next(const DuoParams& p, Stream& s, int lane, int& j,
                                            bool& first, bool& last, int* bad) {
  while (s.live) {
    while (s.r < s.count) {
      const int jj = stream_entry(s, s.r, lane);
      ++s.r;
      if (jj >= 0 && jj <= s.i) {
        j = jj;
        first = s.b == 0;
        ++s.b;
        last = s.b == s.valid;
        return true;
      }
      ++*bad;
    }
    stream_open(p, s, s.t + 2, lane);
  }
  return false;
}

__device__ __forceinline__ void record(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attend_duo_kernel(const __grid_constant__ DuoParams p) {
  using C = DC<D>;
  constexpr int BM = C::BM, BN = C::BN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bar;
  uint64_t* q_full = kv_full + kStages;  // [slot]
  uint64_t* q_free = q_full + 2;         // [slot]
  uint64_t* s_full = q_free + 2;         // [slot][kSBars]
  uint64_t* p_full = s_full + 2 * kSBars;  // [slot]
  uint64_t* o_full = p_full + 2;         // [slot]
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sKV = smem + C::OFF_KV;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&kv_full[s], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_free[x], 1);
      for (int b = 0; b < kSBars; ++b) mbar_init(&s_full[x * kSBars + b], 1);
      mbar_init(&p_full[x], 128);
      mbar_init(&o_full[x], 1);
    }
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
  auto warp_ok = [&](bool v) { return __shfl_sync(0xFFFFFFFFu, v, 0); };

  if (warp == 0) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    Stream st0, st1;
    stream_open(p, st0, 0, lane);
    stream_open(p, st1, 1, lane);
    bool has_prev[2] = {false, false};
    int prev_j[2] = {0, 0}, prev_g[2] = {0, 0};
    int k_cnt[2] = {0, 0};     // S products of the slot so far
    int q_cnt[2] = {0, 0};     // Q tiles loaded for the slot so far
    int pos = 0, bad = 0;
    bool ok = true;
    // what releases the tiles of the last kStages positions, oldest first
    // (lane 0; shifted at every load, so that no array is indexed at run time)
    uint64_t* rel_bar[kStages] = {};
    uint32_t rel_par[kStages] = {};
    // lane 0: copy block j of kv head g of map m into the next ring position
    // (pos, advanced here), once the tile it replaces (position pos - kStages)
    // has been released.  pos is kept by lane 0 only.
    auto load_kv = [&](const CUtensorMap* m, int j, int g, uint64_t* rb, uint32_t rp) -> bool {
      const int s = pos % kStages;
      if (pos >= kStages && !wait(rel_bar[0], rel_par[0])) return false;
#pragma unroll
      for (int q = 0; q + 1 < kStages; ++q) {
        rel_bar[q] = rel_bar[q + 1];
        rel_par[q] = rel_par[q + 1];
      }
      rel_bar[kStages - 1] = rb;
      rel_par[kStages - 1] = rp;
      mbar_arrive_expect_tx(&kv_full[s], C::KV_BYTES);
      for (int a = 0; a < C::NA_D; ++a)
        tma_load_3d(sKV + s * C::KV_BYTES + a * (BN * 128), m, &kv_full[s], a * 64, j * BN, g);
      ++pos;
      return true;
    };
    // one step of slot x (the V tile of its previous block, then the K tile
    // of its next one); inlined once per slot so the cursors stay in registers
    auto step = [&](Stream& sx, const int x) {
      int j = 0;
      bool first = false, last = false;
      const bool found = sx.live && stream_next(p, sx, lane, j, first, last, &bad);
      bool good = true;
      if (lane == 0) {
        // both positions of the step are released by the commit of this
        // step's S product, or, at the end of the slot's stream, by the
        // commit that hands the slot's last O to its epilogue
        uint64_t* rb = found ? &s_full[x * kSBars + k_cnt[x] % kSBars] : &o_full[x];
        const uint32_t rp = found ? (uint32_t)((k_cnt[x] / kSBars) & 1)
                                  : (uint32_t)((q_cnt[x] - 1) & 1);
        if (has_prev[x]) good = load_kv(&p.tm_v, prev_j[x], prev_g[x], rb, rp);
        if (good && found && first) {
          // the slot's Q buffer is free once its previous item's last S is done
          if (q_cnt[x] >= 1) good = wait(&q_free[x], (q_cnt[x] - 1) & 1);
          if (good) {
            mbar_arrive_expect_tx(&q_full[x], C::Q_BYTES);
            for (int a = 0; a < C::NA_D; ++a)
              tma_load_3d(sQ + x * C::Q_BYTES + a * (BM * 128), &p.tm_q, &q_full[x], a * 64,
                          sx.i * BM, sx.h);
          }
        }
        if (good && found) good = load_kv(&p.tm_k, j, sx.g, rb, rp);
      }
      if (!warp_ok(good)) {
        ok = false;
        return;
      }
      if (found) {
        if (first) ++q_cnt[x];
        ++k_cnt[x];
      }
      has_prev[x] = found;
      prev_j[x] = j;
      prev_g[x] = sx.g;
    };
    while (ok) {
      bool any = false;
      if (has_prev[0] || st0.live) {
        any = true;
        step(st0, 0);
      }
      if (ok && (has_prev[1] || st1.live)) {
        any = true;
        step(st1, 1);
      }
      if (!any) break;
    }
    if (lane == 0) {
      if (bad) record(p.status, SBSA_ERR_DEVICE);
      volatile int never = 0;
      const int first = pos > kStages ? pos - kStages : 0;
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        // copies may still be landing in shared memory
        for (int x = 0; x < 2; ++x)
          if (q_cnt[x] > 0) mbar_wait_bounded(&q_full[x], (q_cnt[x] - 1) & 1, &never, kTimeoutNs);
        for (int q = first; q < pos; ++q)
          mbar_wait_bounded(&kv_full[q % kStages], (q / kStages) & 1, &never, kTimeoutNs);
      } else {
        // the last positions are consumed by products whose commits follow
        // (the shift register holds them in its last pos - first entries)
#pragma unroll
        for (int q = 0; q < kStages; ++q)
          if (q >= kStages - (pos - first) && !wait(rel_bar[q], rel_par[q])) break;
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    const uint32_t q_base = smem_u32(sQ);
    const uint32_t kv_base = smem_u32(sKV);
    const uint64_t q_desc0 = smem_desc(q_base, 16, 1024);
    const uint64_t k_desc0 = smem_desc(kv_base, 16, 1024);
    const uint64_t v_desc0 = smem_desc(kv_base, BN * 128, 1024);
    Stream st0, st1;
    stream_open(p, st0, 0, lane);
    stream_open(p, st1, 1, lane);
    bool has_prev[2] = {false, false}, prev_first[2] = {false, false}, prev_last[2] = {false, false};
    int k_cnt[2] = {0, 0};   // S products issued per slot
    int pv_cnt[2] = {0, 0};  // PV products issued per slot
    int q_cnt[2] = {0, 0};   // items started per slot
    int pos = 0, bad = 0;
    bool ok = true, issued = false;
    // one step of slot x (O_x += P_x V for its previous block, then S_x for
    // its next one); inlined once per slot so the cursors stay in registers
    auto step = [&](Stream& sx, const int x) {
      int j = 0;
      bool first = false, last = false;
      const bool found = sx.live && stream_next(p, sx, lane, j, first, last, &bad);
      bool good = true;
      const int vpos = pos;
      const int kpos = pos + (has_prev[x] ? 1 : 0);
      if (lane == 0) {
        if (has_prev[x]) {
          // O_x += P_x V once the softmax has written P
          good = wait(&p_full[x], pv_cnt[x] & 1);
          const int s = vpos % kStages;
          if (good) good = wait(&kv_full[s], (vpos / kStages) & 1);
          if (good) {
            tc_fence_after();
            const uint64_t bd0 = v_desc0 + (uint64_t)(s * (C::KV_BYTES >> 4));
            const uint32_t a_col = tmem + C::TM_S + x * BN;
            const uint32_t o_col = tmem + C::TM_O + x * D;
            const uint32_t acc0 = prev_first[x] ? 0u : 1u;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              umma_f16_ts(o_col, a_col + kk * 8, bd0 + (uint64_t)(kk * 128), C::IDESC_O,
                          kk > 0 ? 1u : acc0);
            if (prev_last[x]) umma_commit(&o_full[x]);
            issued = true;
          }
        }
        if (good && found) {
          // S_x = Q_x K^T
          if (first) good = wait(&q_full[x], q_cnt[x] & 1);
          const int s = kpos % kStages;
          if (good) good = wait(&kv_full[s], (kpos / kStages) & 1);
          if (good) {
            tc_fence_after();
            const uint64_t ad0 = q_desc0 + (uint64_t)(x * (C::Q_BYTES >> 4));
            const uint64_t bd0 = k_desc0 + (uint64_t)(s * (C::KV_BYTES >> 4));
            const uint32_t s_col = tmem + C::TM_S + x * BN;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // 32 bytes per K-step inside a 128-byte swizzle atom, then the
              // next atom (BM or BN rows of 128 bytes) every 4 steps
              const int kb = kk * 32;
              const uint64_t da = (uint64_t)(((kb / 128) * (BM * 128) + (kb % 128)) >> 4);
              const uint64_t db = (uint64_t)(((kb / 128) * (BN * 128) + (kb % 128)) >> 4);
              umma_f16_ss(s_col, ad0 + da, bd0 + db, C::IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[x * kSBars + k_cnt[x] % kSBars]);
            if (last) umma_commit(&q_free[x]);
            issued = true;
          }
        }
      }
      if (!warp_ok(good)) {
        ok = false;
        return;
      }
      if (has_prev[x]) {
        ++pv_cnt[x];
        ++pos;
      }
      if (found) {
        if (first) ++q_cnt[x];
        ++k_cnt[x];
        ++pos;
      }
      has_prev[x] = found;
      prev_first[x] = first;
      prev_last[x] = last;
    };
    while (ok) {
      bool any = false;
      if (has_prev[0] || st0.live) {
        any = true;
        step(st0, 0);
      }
      if (ok && (has_prev[1] || st1.live)) {
        any = true;
        step(st1, 1);
      }
      if (!any) break;
    }
    if (lane == 0 && !ok) {
      if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
      if (issued) {
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait_bounded(drain, 0, &never, kTimeoutNs);
      }
    }
  } else {
    // ================================================================ softmax
    const int x = (warp - 2) >> 2;       // slot
    const int qd = warp & 3;             // TMEM lane quadrant
    const int row = qd * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const uint32_t s_col = tmem + lane_base + C::TM_S + x * BN;
    const uint32_t o_col = tmem + lane_base + C::TM_O + x * D;
    int kk_s = 0;        // S blocks consumed
    int items_done = 0;  // items with products, finished
    bool ok = true;
    Stream it;
    for (int t = x; ok && stream_open(p, it, t, lane); t += 2) {
      const int tok = it.i * BM + row;
      const bool store = tok < p.n;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)it.h * p.n + tok) * D;
      if (it.valid == 0) {
        // nothing listed: the output rows are zero
        if (store) {
#pragma unroll
          for (int c = 0; c < D; c += 8)
            *reinterpret_cast<uint4*>(orow + c) = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;
      int b = 0;
      for (int r = 0; r < it.count; ++r) {
        const int j = stream_entry(it, r, lane);
        if (!(j >= 0 && j <= it.i)) continue;
        const bool diag = (j == it.i);
        if (!wait(&s_full[x * kSBars + kk_s % kSBars], (kk_s / kSBars) & 1)) ok = false;
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        ++kk_s;
        tc_fence_after();
        // keys past `lim` are masked (the causal triangle of the diagonal
        // block); one code path for every block keeps the kernel's code small
        const int lim = diag ? row : BN - 1;
        // pass 1: the row maximum over the 128 scores
        float mx = -INFINITY;
        {
          float su[4][32];
          tmem_ld32(s_col + 0, su[0]);
          tmem_ld32(s_col + 32, su[1]);
          tmem_ld32(s_col + 64, su[2]);
          tmem_ld32(s_col + 96, su[3]);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < 32; ++c) mx = fmaxf(mx, 32 * u + c <= lim ? su[u][c] : -INFINITY);
        }
        // the running maximum moves only when the row maximum exceeds it by
        // more than 2^8 (in any row of the warp); O is rescaled below, after
        // P has been written
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        float alpha = 1.f;
        bool rescale = false;
        if (b == 0) {
          m_run = m_new;
        } else if (__any_sync(0xFFFFFFFFu, m_new > m_run + kRescaleLog2)) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
          rescale = true;
        }
        // pass 2: P = exp2(S * scale - m) as bf16 over the first half of the
        // S columns, 64 keys at a time: keys [64h, 64h + 64) -> columns
        // [32h, 32h + 32) (P's first half overwrites keys 0-63 only after
        // they were read)
        float lsum = 0.f;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          float a0[32], a1[32];
          tmem_ld32(s_col + hh * 64, a0);
          tmem_ld32(s_col + hh * 64 + 32, a1);
          tmem_wait_ld();
          const int lh = lim - hh * 64;
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float p0 = ex2_approx(fmaf(a0[c], p.scale_log2, -m_run));
            float p1 = ex2_approx(fmaf(a0[c + 1], p.scale_log2, -m_run));
            float p2 = ex2_approx(fmaf(a1[c], p.scale_log2, -m_run));
            float p3 = ex2_approx(fmaf(a1[c + 1], p.scale_log2, -m_run));
            p0 = c <= lh ? p0 : 0.f;
            p1 = c + 1 <= lh ? p1 : 0.f;
            p2 = c + 32 <= lh ? p2 : 0.f;
            p3 = c + 33 <= lh ? p3 : 0.f;
            lsum += (p0 + p1) + (p2 + p3);
            pk[c >> 1] = pack_bf16x2(p0, p1);
            pk[16 + (c >> 1)] = pack_bf16x2(p2, p3);
          }
          tmem_st32u(s_col + hh * 32, pk);
        }
        if (rescale) {
          // the commit that announced this S also covers the slot's previous
          // PV, so O is quiescent here; this block's PV waits for p_full
          l_run *= alpha;
#pragma unroll 1
          for (int oc = 0; oc < D; oc += 16) {
            float o[16];
            tmem_ld16(o_col + oc, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= alpha;
            tmem_st16(o_col + oc, o);
          }
        }
        l_run += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[x]);
        ++b;
      }
      if (!ok) break;
      // epilogue: O / l of this item
      if (!wait(&o_full[x], items_done & 1)) ok = false;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      ++items_done;
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tmem_ld32(o_col + c0, o);
        tmem_wait_ld();
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
  using C = DC<D>;
  DuoParams p{};
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&p.tm_q, dt, 2, a.q, a.hq, a.n, D, 128) ||
      !make_map(&p.tm_k, dt, 2, a.k, a.hkv, a.n, D, 128) ||
      !make_map(&p.tm_v, dt, 2, a.v, a.hkv, a.n, D, 128))
    return SBSA_ERR_CUDA;
  p.o = a.o;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.hq = a.hq;
  p.n = a.n;
  p.nb = (a.n + 127) / 128;
  p.group = a.hq / a.hkv;
  p.kmax = a.kmax;
  p.total = (long long)a.hq * p.nb;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.status = a.status;
  auto kern = attend_duo_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SBSA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return SBSA_ERR_CUDA;
  const int grid = p.total < sms ? (int)p.total : sms;
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SBSA_OK : SBSA_ERR_CUDA;
}

}  // namespace

int launch_attend_duo(const AttendArgs& a, cudaStream_t stream) {
  if (a.dtype != SBSA_BF16 || a.block != 128 || a.group_shared) return SBSA_ERR_UNSUPPORTED;
  if (a.d == 128) return launch_d<128>(a, stream);
  if (a.d == 64) return launch_d<64>(a, stream);
  return SBSA_ERR_UNSUPPORTED;
}

}  // namespace sbsa
