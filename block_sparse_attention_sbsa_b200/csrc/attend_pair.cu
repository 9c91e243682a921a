// Attention over the selected key blocks for two query heads of one GQA
// group at once (bf16, 128-token blocks).
//
// "RBS-Attention" (iaonda.com), method paragraph: sparse prefill compatible
// with sparse FlashAttention, i.e. exact softmax attention restricted to the
// kept blocks.  "MiniMax presenta MSA", "Que es MSA y como funciona?": one
// block selection shared by a GQA group, full attention over those blocks.
//
// A work item is a query block i and a pair of query heads (h, h + 1) that
// read the same kv head.  The kernel walks the ascending union of the two
// heads' lists and loads each K_j / V_j tile into shared memory once for both
// query tiles; a block in one list only is multiplied for that tile only.
// Shared lists (one per GQA group) and overlapping per-head lists (diagonal
// and rescued blocks) thus halve or reduce the K/V traffic per product.
//
// One CTA per SM walks a static, longest-first list of items.  10 warps:
//   warp 0     TMA producer: Q_A, Q_B of each item (once the previous item's
//              products are done); K_j, V_j of the union list into a 5-stage
//              ring.
//   warp 1     TMEM owner and single-thread MMA issuer: per union block, in
//              order S_A = Q_A K^T, S_B = Q_B K^T, then (once the softmax has
//              written P over the first half of S in TMEM) O_A += P_A V and
//              O_B += P_B V, interleaved so each tile's next product waits only
//              for its own softmax.
//   warps 2-5  softmax and epilogue of tile A, warps 6-9 of tile B: one row
//              per thread over its own list; the running maximum is moved
//              (and O rescaled in TMEM) only when it grows by more than 2^8;
//              the commit that announces S covers the tile's previous PV, so
//              O is quiescent when rescaled.
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
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct PC {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int NA_D = D / 64;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;                     // Q[tile]
  static constexpr int OFF_KV = 2 * Q_BYTES;          // ring[kStages]
  static constexpr int OFF_BAR = OFF_KV + kStages * KV_BYTES;
  // q_full q_free kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2]
  // o_free[2] drain   (s/p/o barriers per tile)
  static constexpr int NBARS = 1 + 1 + 2 * kStages + 2 + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S = 0;       // S[tile]: BN columns each
  static constexpr int TM_O = 2 * BN;  // O[tile]: D columns each
  static constexpr int TM_COLS = 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, BM, BN, false, false);
  static constexpr uint32_t IDESC_O = make_idesc(1, BM, D, false, true);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(2 * BN + 2 * D <= TM_COLS, "TMEM budget");
};

struct PCParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void* o;
  const int32_t* idx;
  const int32_t* cnt;
  int hq, n, nb, group, group_shared, kmax, pairs, total;
  float scale_log2;
  int* status;
};

// One head's list, read by a whole warp: lane l holds entry base + l.
struct List {
  const int32_t* ptr;
  int count;
  int base;
  int val;
};

__device__ __forceinline__ void list_open(List& L, const int32_t* ptr, int count, int lane) {
  L.ptr = ptr;
  L.count = count;
  L.base = 0;
  L.val = lane < count ? ptr[lane] : -1;
}

__device__ __forceinline__ int list_at(List& L, int r, int lane) {
  const int base = r & ~31;
  if (base != L.base) {
    L.base = base;
    L.val = base + lane < L.count ? L.ptr[base + lane] : -1;
  }
  return __shfl_sync(0xFFFFFFFFu, L.val, r & 31);
}

struct Item {
  int i, hA, g;    // query block, first head of the pair, kv head
  List a, b;       // the two heads' lists
  int ra, rb;      // cursors of the union walk
};

__device__ __forceinline__ bool open_item(const PCParams& p, int t, Item& it, int lane) {
  const long long item = (long long)blockIdx.x + (long long)t * gridDim.x;
  if (item >= p.total) return false;
  it.i = p.nb - 1 - (int)(item / p.pairs);
  const int pr = (int)(item % p.pairs);
  it.hA = 2 * pr;
  it.g = it.hA / p.group;
  const int hsA = p.group_shared ? it.g : it.hA;
  const int hsB = p.group_shared ? it.g : it.hA + 1;
  const int32_t* la = p.idx + ((size_t)hsA * p.nb + it.i) * p.kmax;
  const int32_t* lb = p.idx + ((size_t)hsB * p.nb + it.i) * p.kmax;
  int ca = p.cnt[(size_t)hsA * p.nb + it.i];
  int cb = p.cnt[(size_t)hsB * p.nb + it.i];
  ca = ca < 0 ? 0 : (ca > p.kmax ? p.kmax : ca);
  cb = cb < 0 ? 0 : (cb > p.kmax ? p.kmax : cb);
  list_open(it.a, la, ca, lane);
  list_open(it.b, lb, cb, lane);
  it.ra = 0;
  it.rb = 0;
  return true;
}

__device__ __forceinline__ bool in_range(int j, int i) { return j >= 0 && j <= i; }

// Next block of the ascending union of the two lists; entries outside
// [0, i] are skipped (and counted in *bad).  Returns false at the end.
__device__ __forceinline__ bool union_next(Item& it, int lane, int& j, bool& inA, bool& inB,
                                           int* bad) {
  int ja = -1, jb = -1;
  while (it.ra < it.a.count) {
    ja = list_at(it.a, it.ra, lane);
    if (in_range(ja, it.i)) break;
    ++*bad;
    ++it.ra;
    ja = -1;
  }
  while (it.rb < it.b.count) {
    jb = list_at(it.b, it.rb, lane);
    if (in_range(jb, it.i)) break;
    ++*bad;
    ++it.rb;
    jb = -1;
  }
  const bool ha = it.ra < it.a.count, hb = it.rb < it.b.count;
  if (!ha && !hb) return false;
  if (ha && (!hb || ja <= jb)) {
    j = ja;
    inA = true;
    inB = hb && jb == ja;
  } else {
    j = jb;
    inA = false;
    inB = true;
  }
  if (inA) ++it.ra;
  if (inB) ++it.rb;
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
__global__ void __launch_bounds__(kThreads, 1) attend_pair_kernel(const __grid_constant__ PCParams p) {
  using C = PC<D>;
  constexpr int BM = C::BM, BN = C::BN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* q_free = q_full + 1;
  uint64_t* kv_full = q_free + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;  // [tile]
  uint64_t* p_full = s_full + 2;          // [tile]
  uint64_t* o_full = p_full + 2;          // [tile]
  uint64_t* o_free = o_full + 2;          // [tile]
  uint64_t* drain = o_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sKV = smem + C::OFF_KV;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], 128);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
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
    // Two cursors: the K/V cursor walks the union lists item after item (the
    // next item's tiles stream in while the current item still computes);
    // the Q cursor loads an item's two Q tiles once the previous item's
    // products are done with the single Q buffer.  Both are polled without
    // blocking; a stretch of 2 s without progress counts as a timeout.
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    int pos = 0, bad = 0, kv_t = 0, q_t = 0, half = 0, jcur = 0;
    bool have_j = false, ok = true;
    Item kv_it, q_it;
    bool kv_live = open_item(p, 0, kv_it, lane);
    bool q_live = open_item(p, 0, q_it, lane);
    uint64_t t_last = global_timer_ns();
    while (kv_live || q_live) {
      bool progress = false;
      if (q_live && q_t <= kv_t) {
        bool go = true;
        if (lane == 0) {
          go = q_t == 0 || mbar_test_wait(q_free, (q_t - 1) & 1);
          if (go) {
            mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
            for (int tile = 0; tile < 2; ++tile)
              for (int a = 0; a < C::NA_D; ++a)
                tma_load_3d(sQ + tile * C::Q_BYTES + a * (BM * 128), &p.tm_q, q_full, a * 64,
                            q_it.i * BM, q_it.hA + tile);
          }
        }
        if (__shfl_sync(0xFFFFFFFFu, go, 0)) {
          ++q_t;
          q_live = open_item(p, q_t, q_it, lane);
          progress = true;
        }
      }
      if (kv_live) {
        if (!have_j) {
          bool inA, inB;
          have_j = union_next(kv_it, lane, jcur, inA, inB, &bad);
          half = 0;
          if (!have_j) {
            ++kv_t;
            kv_live = open_item(p, kv_t, kv_it, lane);
            progress = true;
          }
        }
        if (have_j) {
          const int st = pos % kStages;
          bool go = true;
          if (lane == 0) {
            go = mbar_test_wait(&kv_empty[st], ((pos / kStages) & 1) ^ 1);
            if (go) {
              mbar_arrive_expect_tx(&kv_full[st], C::KV_BYTES);
              const CUtensorMap* m = half ? &p.tm_v : &p.tm_k;
              for (int a = 0; a < C::NA_D; ++a)
                tma_load_3d(sKV + st * C::KV_BYTES + a * (BN * 128), m, &kv_full[st], a * 64,
                            jcur * BN, kv_it.g);
            }
          }
          if (__shfl_sync(0xFFFFFFFFu, go, 0)) {
            ++pos;
            if (half) have_j = false;
            half ^= 1;
            progress = true;
          }
        }
      }
      bool stop = false;
      if (lane == 0) {
        if (progress) {
          t_last = global_timer_ns();
        } else {
          __nanosleep(64);
          stop = *abort_flag || global_timer_ns() - t_last > kTimeoutNs;
        }
      }
      if (__shfl_sync(0xFFFFFFFFu, stop, 0)) {
        ok = false;
        break;
      }
    }
    if (lane == 0) {
      if (bad) record(p.status, SBSA_ERR_DEVICE);
      volatile int never = 0;
      const int first = pos > kStages ? pos - kStages : 0;
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        // copies may still be landing in shared memory
        if (q_t > 0) mbar_wait_bounded(q_full, (q_t - 1) & 1, &never, kTimeoutNs);
        for (int q = first; q < pos; ++q)
          mbar_wait_bounded(&kv_full[q % kStages], (q / kStages) & 1, &never, kTimeoutNs);
      } else {
        // wait for the MMA thread's last asynchronous releases
        for (int q = first; q < pos; ++q)
          if (!wait(&kv_empty[q % kStages], (q / kStages) & 1)) break;
        if (q_t > 0) wait(q_free, (q_t - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    const uint32_t q_base = smem_u32(sQ);
    const uint32_t kv_base = smem_u32(sKV);
    // per tile: PVs issued so far and the PV still pending (its V ring
    // position, whether it starts the tile's item, and the item)
    int p_cnt[2] = {0, 0};
    int pend_pos[2] = {-1, -1};
    int pend_first[2] = {0, 0};
    int pend_t[2] = {0, 0};
    // PVs still to be issued for the V stage of each of the last 4 blocks
    int v_left[4] = {0, 0, 0, 0};
    bool ok = true;
    int pos = 0, t = 0, bad = 0;
    Item it;
    // lane 0: issue the pending PV of `tile` (waits for its P); the V stage
    // is released after the last PV that reads it
    auto issue_pv = [&](int tile) -> bool {
      if (pend_pos[tile] < 0) return true;
      if (!wait(&p_full[tile], p_cnt[tile] & 1)) return false;
      const int tt = pend_t[tile];
      if (pend_first[tile] && tt >= 1 && !wait(&o_free[tile], (tt - 1) & 1)) return false;
      const int vpos = pend_pos[tile];
      const int st = vpos % kStages;
      if (!wait(&kv_full[st], (vpos / kStages) & 1)) return false;
      tc_fence_after();
      const uint32_t v_base = kv_base + st * C::KV_BYTES;
      const uint32_t a_col = tmem + C::TM_S + tile * BN;
      const uint32_t o_col = tmem + C::TM_O + tile * D;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const uint64_t bd = smem_desc(v_base + kk * 16 * 128, BN * 128, 1024);
        umma_f16_ts(o_col, a_col + kk * 8, bd, C::IDESC_O,
                    (!pend_first[tile] || kk > 0) ? 1u : 0u);
      }
      if (--v_left[(vpos >> 1) & 3] == 0) umma_commit(&kv_empty[st]);
      ++p_cnt[tile];
      pend_pos[tile] = -1;
      return true;
    };
    for (; ok && open_item(p, t, it, lane); ++t) {
      bool good = true;
      if (lane == 0) {
        good = wait(q_full, t & 1);
        if (good) tc_fence_after();
      }
      if (!warp_ok(good)) {
        ok = false;
        break;
      }
      bool first[2] = {true, true};
      int j;
      bool in[2];
      while (union_next(it, lane, j, in[0], in[1], &bad)) {
        const int kpos = pos, vpos = pos + 1;
        pos += 2;
        if (lane == 0) {
          const int kst = kpos % kStages;
          v_left[(vpos >> 1) & 3] = (in[0] ? 1 : 0) + (in[1] ? 1 : 0);
          good = wait(&kv_full[kst], (kpos / kStages) & 1);
          if (good) {
            tc_fence_after();
            const uint32_t ka = kv_base + kst * C::KV_BYTES;
            for (int tile = 0; tile < 2 && good; ++tile) {
              if (!in[tile]) continue;
              // the tile's previous PV reads P from the S columns: issue it first
              good = issue_pv(tile);
              if (!good) break;
              const uint32_t qa = q_base + tile * C::Q_BYTES;
              const uint32_t s_col = tmem + C::TM_S + tile * BN;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const int kb = kk * 32;
                const uint64_t ad = smem_desc(qa + (kb / 128) * (BM * 128) + (kb % 128), 16, 1024);
                const uint64_t bd = smem_desc(ka + (kb / 128) * (BN * 128) + (kb % 128), 16, 1024);
                umma_f16_ss(s_col, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
              }
              umma_commit(&s_full[tile]);
              pend_pos[tile] = vpos;
              pend_first[tile] = first[tile] ? 1 : 0;
              pend_t[tile] = t;
              first[tile] = false;
            }
            if (good) umma_commit(&kv_empty[kst]);
            // a tile absent from this block issues its pending PV now, so no
            // V stage stays pinned while the other tile moves on
            for (int tile = 0; tile < 2 && good; ++tile)
              if (!in[tile] && pend_pos[tile] >= 0) good = issue_pv(tile);
          }
        }
        if (!warp_ok(good)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      // end of item: issue both pending PVs, hand O to the epilogues and
      // release the Q tiles
      if (lane == 0) {
        for (int tile = 0; tile < 2 && good; ++tile) good = issue_pv(tile);
        if (good) {
          for (int tile = 0; tile < 2; ++tile) umma_commit(&o_full[tile]);
          umma_commit(q_free);
        }
      }
      if (!warp_ok(good)) {
        ok = false;
        break;
      }
    }
    if (lane == 0 && !ok) {
      if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait_bounded(drain, 0, &never, kTimeoutNs);
    }
  } else {
    // ================================================================ softmax
    const int tile = (warp - 2) >> 2;
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const uint32_t s_col = tmem + lane_base + C::TM_S + tile * BN;
    const uint32_t o_col = tmem + lane_base + C::TM_O + tile * D;
    int scnt = 0;
    bool ok = true;
    Item it;
    for (int t = 0; ok && open_item(p, t, it, lane); ++t) {
      List& L = tile ? it.b : it.a;
      float m_run = -INFINITY, l_run = 0.f;
      int b = 0;
      for (int r = 0; r < L.count; ++r) {
        const int j = list_at(L, r, lane);
        if (!in_range(j, it.i)) continue;
        const bool diag = (j == it.i);
        if (!wait(&s_full[tile], scnt & 1)) ok = false;
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        ++scnt;
        tc_fence_after();
        // pass 1: row maximum (64 columns at a time)
        float mx = -INFINITY;
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float a[32], bb[32];
          tmem_ld32(s_col + c0, a);
          tmem_ld32(s_col + c0 + 32, bb);
          tmem_wait_ld();
          if (diag) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c0 + c <= row) mx = fmaxf(mx, a[c]);
              if (c0 + 32 + c <= row) mx = fmaxf(mx, bb[c]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(a[c], bb[c]));
          }
        }
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        if (b == 0) {
          m_run = m_new;
        } else if (__any_sync(0xFFFFFFFFu, m_new > m_run + kRescaleLog2)) {
          // the commit announcing this S covers the tile's previous PV
          const float alpha = ex2_approx(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
#pragma unroll
          for (int oc = 0; oc < D; oc += 16) {
            float o[16];
            tmem_ld16(o_col + oc, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= alpha;
            tmem_st16(o_col + oc, o);
          }
        }
        // pass 2: P = exp2(S * scale - m) as bf16 over the first half of the
        // S columns (step c0 reads S[c0, c0+64), writes P to [c0/2, c0/2+32));
        // the two steps stay a loop: unrolled, the kernel spills
        float lsum = 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float a[32], bb[32];
          tmem_ld32(s_col + c0, a);
          tmem_ld32(s_col + c0 + 32, bb);
          tmem_wait_ld();
          if (diag) {
            // causal mask of the diagonal block: keys past the row's own
            // token score -inf, so the exponentials need no test of their
            // own (exp2(-inf) = +0)
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c0 + c > row) a[c] = -INFINITY;
              if (c0 + 32 + c > row) bb[c] = -INFINITY;
            }
          }
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = ex2_approx(fmaf(a[c], p.scale_log2, -m_run));
            const float p1 = ex2_approx(fmaf(a[c + 1], p.scale_log2, -m_run));
            const float p2 = ex2_approx(fmaf(bb[c], p.scale_log2, -m_run));
            const float p3 = ex2_approx(fmaf(bb[c + 1], p.scale_log2, -m_run));
            lsum += (p0 + p1) + (p2 + p3);
            pk[c >> 1] = pack_bf16x2(p0, p1);
            pk[16 + (c >> 1)] = pack_bf16x2(p2, p3);
          }
          tmem_st32u(s_col + (c0 >> 1), pk);
        }
        l_run += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[tile]);
        ++b;
      }
      if (!ok) break;
      // epilogue of this tile's item
      if (!wait(&o_full[tile], t & 1)) ok = false;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int h = it.hA + tile;
      const int tok = it.i * BM + row;
      const bool store = tok < p.n;
      const float inv_l = (b > 0 && l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)h * p.n + tok) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        if (b > 0) {
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
      mbar_arrive(&o_free[tile]);
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
  using C = PC<D>;
  PCParams p{};
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
  p.group_shared = a.group_shared;
  p.kmax = a.kmax;
  p.pairs = a.hq / 2;
  p.total = p.pairs * p.nb;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.status = a.status;
  auto kern = attend_pair_kernel<D>;
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

int launch_attend_pair(const AttendArgs& a, cudaStream_t stream) {
  if (a.dtype != SBSA_BF16 || a.block != 128 || (a.hq / a.hkv) % 2 != 0)
    return SBSA_ERR_UNSUPPORTED;
  if (a.d == 128) return launch_d<128>(a, stream);
  if (a.d == 64) return launch_d<64>(a, stream);
  return SBSA_ERR_UNSUPPORTED;
}

}  // namespace sbsa
