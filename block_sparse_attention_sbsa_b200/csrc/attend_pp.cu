// Attention over the selected key blocks, persistent two-tile version for
// bf16 with 128-token blocks (the long-context workloads).
//
// "RBS-Attention" (iaonda.com), method paragraph: sparse prefill compatible
// with sparse FlashAttention, i.e. exact softmax attention restricted to the
// kept blocks.  "MiniMax presenta MSA", "Que es MSA y como funciona?": full
// attention over the preselected blocks only.
//
// One CTA per SM walks a static list of (query head, query block) work items
// (longest lists first).  Two items are in flight at a time, one per slot,
// so the tensor core computes one slot's products while the other slot's
// softmax runs.  10 warps:
//   warp 0      TMA producer for both slots (Q tile per item, K_j / V_j
//               tiles into a 2-stage ring per slot), non-blocking polling.
//   warp 1      TMEM owner and single-thread MMA issuer, polling both slots:
//               S = Q K_j^T into the slot's S columns; after the softmax has
//               written P (bf16) over the first half of those columns,
//               O += P V_j with P read from tensor memory.
//   warps 2-5   softmax of slot 0, warps 6-9 softmax of slot 1: one query row
//               per thread, running maximum moved (and O rescaled in TMEM)
//               only when it grows by more than 2^8, epilogue O / l.
// Per slot the MMAs run in issue order S(0), PV(0), S(1), PV(1), ...; the
// commit after S(n) therefore also covers PV(n-1), so when the softmax sees
// S(n) the slot's O is quiescent and may be rescaled.
// Every wait is bounded: a role that sees no progress for 2 s records
// SBSA_ERR_TIMEOUT, raises the CTA's abort flag, drains what it issued and
// leaves; TMEM is freed by the owner warp at the end.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "tma_map.h"

namespace sbsa {
namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kSlots = 2;
constexpr int kStages = 2;  // K/V ring stages per slot (K in stage 0, V in stage 1)
constexpr int kThreads = 320;
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct PP {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int NA_D = D / 64;  // 128-byte swizzle atoms across d (bf16)
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = kSlots * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + kSlots * kStages * KV_BYTES;
  static constexpr int BARS_PER_SLOT = 10;
  static constexpr int NBARS = kSlots * BARS_PER_SLOT + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_SLOT = BN + D;  // S (P over its first BN/2 columns), then O
  static constexpr int TM_COLS = 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, BM, BN, false, false);
  static constexpr uint32_t IDESC_O = make_idesc(1, BM, D, false, true);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(kSlots * TM_SLOT <= TM_COLS, "TMEM budget");
};

struct PPParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void* o;
  const int32_t* idx;
  const int32_t* cnt;
  int hq, n, nb, group, group_shared, kmax, total;
  float scale_log2;
  int* status;
};

struct Item {
  int i, h, g, count;
  const int32_t* list;
};

__device__ __forceinline__ bool load_item(const PPParams& p, int slot, int ordinal, Item& it) {
  const int k = slot + 2 * ordinal;
  const long long item = (long long)blockIdx.x + (long long)k * gridDim.x;
  if (item >= p.total) return false;
  it.i = p.nb - 1 - (int)(item / p.hq);
  it.h = (int)(item % p.hq);
  it.g = it.h / p.group;
  const int hs = p.group_shared ? it.g : it.h;
  it.list = p.idx + ((size_t)hs * p.nb + it.i) * p.kmax;
  int c = p.cnt[(size_t)hs * p.nb + it.i];
  it.count = c < 0 ? 0 : (c > p.kmax ? p.kmax : c);
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
__global__ void __launch_bounds__(kThreads, 1) attend_pp_kernel(const __grid_constant__ PPParams p) {
  using C = PP<D>;
  constexpr int BM = C::BM, BN = C::BN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // per slot X: q_full, q_free, kv_full[2], kv_empty[2], s_full, p_full, o_full, o_free
  auto q_full = [&](int X) { return bars + X * C::BARS_PER_SLOT + 0; };
  auto q_free = [&](int X) { return bars + X * C::BARS_PER_SLOT + 1; };
  auto kv_full = [&](int X, int s) { return bars + X * C::BARS_PER_SLOT + 2 + s; };
  auto kv_empty = [&](int X, int s) { return bars + X * C::BARS_PER_SLOT + 4 + s; };
  auto s_full = [&](int X) { return bars + X * C::BARS_PER_SLOT + 6; };
  auto p_full = [&](int X) { return bars + X * C::BARS_PER_SLOT + 7; };
  auto o_full = [&](int X) { return bars + X * C::BARS_PER_SLOT + 8; };
  auto o_free = [&](int X) { return bars + X * C::BARS_PER_SLOT + 9; };
  uint64_t* drain = bars + kSlots * C::BARS_PER_SLOT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto sQ = [&](int X) { return smem + C::OFF_Q + X * C::Q_BYTES; };
  auto sKV = [&](int X, int s) { return smem + C::OFF_KV + (X * kStages + s) * C::KV_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int X = 0; X < kSlots; ++X) {
      mbar_init(q_full(X), 1);
      mbar_init(q_free(X), 1);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(kv_full(X, s), 1);
        mbar_init(kv_empty(X, s), 1);
      }
      mbar_init(s_full(X), 1);
      mbar_init(p_full(X), 128);
      mbar_init(o_full(X), 1);
      mbar_init(o_free(X), 128);
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

  if (warp == 0) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      // Two cursors per slot: the K/V cursor walks the lists item after item
      // (its next item's tiles may stream in while the current item still
      // computes); the Q cursor loads an item's Q once the slot's previous
      // item has finished with the single Q buffer.
      Item kv_it[kSlots], q_it[kSlots];
      bool kv_live[kSlots], q_live[kSlots];
      int kv_ord[kSlots] = {0, 0}, q_ord[kSlots] = {0, 0};
      int r[kSlots] = {0, 0}, half[kSlots] = {0, 0}, pos[kSlots] = {0, 0};
#pragma unroll
      for (int X = 0; X < kSlots; ++X) {
        kv_live[X] = load_item(p, X, 0, kv_it[X]);
        q_live[X] = load_item(p, X, 0, q_it[X]);
      }
      uint64_t t_last = global_timer_ns();
      bool ok = true;
      while (kv_live[0] || kv_live[1] || q_live[0] || q_live[1]) {
        bool progress = false;
#pragma unroll
        for (int X = 0; X < kSlots; ++X) {
          if (q_live[X] && q_ord[X] <= kv_ord[X] &&
              (q_ord[X] == 0 || mbar_test_wait(q_free(X), (q_ord[X] - 1) & 1))) {
            mbar_arrive_expect_tx(q_full(X), C::Q_BYTES);
            for (int a = 0; a < C::NA_D; ++a)
              tma_load_3d(sQ(X) + a * (BM * 128), &p.tm_q, q_full(X), a * 64, q_it[X].i * BM,
                          q_it[X].h);
            ++q_ord[X];
            q_live[X] = load_item(p, X, q_ord[X], q_it[X]);
            progress = true;
          }
          if (!kv_live[X]) continue;
          while (r[X] < kv_it[X].count) {
            const int j = kv_it[X].list[r[X]];
            if (j >= 0 && j <= kv_it[X].i) break;
            record(p.status, SBSA_ERR_DEVICE);
            ++r[X];
          }
          if (r[X] >= kv_it[X].count) {  // every tile of this item is issued
            ++kv_ord[X];
            kv_live[X] = load_item(p, X, kv_ord[X], kv_it[X]);
            r[X] = 0;
            half[X] = 0;
            progress = true;
            continue;
          }
          const int st = pos[X] & 1;
          if (!mbar_test_wait(kv_empty(X, st), ((pos[X] >> 1) & 1) ^ 1)) continue;
          const int j = kv_it[X].list[r[X]];
          mbar_arrive_expect_tx(kv_full(X, st), C::KV_BYTES);
          const CUtensorMap* m = half[X] ? &p.tm_v : &p.tm_k;
          for (int a = 0; a < C::NA_D; ++a)
            tma_load_3d(sKV(X, st) + a * (BN * 128), m, kv_full(X, st), a * 64, j * BN,
                        kv_it[X].g);
          ++pos[X];
          if (half[X]) ++r[X];
          half[X] ^= 1;
          progress = true;
        }
        if (progress) {
          t_last = global_timer_ns();
        } else if (*abort_flag || global_timer_ns() - t_last > kTimeoutNs) {
          ok = false;
          break;
        }
      }
      volatile int never = 0;
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        // copies may still be landing: wait for each slot's outstanding loads
        for (int X = 0; X < kSlots; ++X) {
          if (q_ord[X] > 0) mbar_wait_bounded(q_full(X), (q_ord[X] - 1) & 1, &never, kTimeoutNs);
          for (int q = pos[X] > kStages ? pos[X] - kStages : 0; q < pos[X]; ++q)
            mbar_wait_bounded(kv_full(X, q & 1), (q >> 1) & 1, &never, kTimeoutNs);
        }
      } else {
        // the MMA thread releases stages and Q with asynchronous commits:
        // wait for the last release of each so none lands after exit
        for (int X = 0; X < kSlots; ++X) {
          for (int q = pos[X] > kStages ? pos[X] - kStages : 0; q < pos[X]; ++q)
            if (!mbar_wait_bounded(kv_empty(X, q & 1), (q >> 1) & 1, abort_flag, kTimeoutNs)) break;
          if (q_ord[X] > 0) mbar_wait_bounded(q_free(X), (q_ord[X] - 1) & 1, abort_flag, kTimeoutNs);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0) {
      Item it[kSlots];
      bool live[kSlots];
      int ord[kSlots] = {0, 0}, r[kSlots] = {0, 0}, nv[kSlots] = {0, 0}, pos[kSlots] = {0, 0};
      int pcnt[kSlots] = {0, 0};
      bool qready[kSlots] = {false, false}, want_pv[kSlots] = {false, false};
#pragma unroll
      for (int X = 0; X < kSlots; ++X) live[X] = load_item(p, X, 0, it[X]);
      uint64_t t_last = global_timer_ns();
      bool ok = true;
      while (live[0] || live[1]) {
        bool progress = false;
#pragma unroll
        for (int X = 0; X < kSlots; ++X) {
          if (!live[X]) continue;
          const uint32_t s_col = tmem + X * C::TM_SLOT;
          const uint32_t o_col = s_col + BN;
          if (!want_pv[X]) {
            // ---- next S = Q K_j^T, or close the item
            if (!qready[X]) {
              if (!mbar_test_wait(q_full(X), ord[X] & 1)) continue;
              qready[X] = true;
            }
            while (r[X] < it[X].count) {
              const int j = it[X].list[r[X]];
              if (j >= 0 && j <= it[X].i) break;
              ++r[X];
            }
            if (r[X] >= it[X].count) {
              umma_commit(q_free(X));
              umma_commit(o_full(X));
              ++ord[X];
              live[X] = load_item(p, X, ord[X], it[X]);
              r[X] = 0;
              nv[X] = 0;
              qready[X] = false;
              progress = true;
              continue;
            }
            const int st = pos[X] & 1;
            if (!mbar_test_wait(kv_full(X, st), (pos[X] >> 1) & 1)) continue;
            tc_fence_after();
            const uint32_t q_base = smem_u32(sQ(X));
            const uint32_t k_base = smem_u32(sKV(X, st));
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int kb = kk * 32;
              const uint64_t ad = smem_desc(q_base + (kb / 128) * (BM * 128) + (kb % 128), 16, 1024);
              const uint64_t bd = smem_desc(k_base + (kb / 128) * (BN * 128) + (kb % 128), 16, 1024);
              umma_f16_ss(s_col, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(kv_empty(X, st));
            umma_commit(s_full(X));
            ++pos[X];
            want_pv[X] = true;
            progress = true;
          } else {
            // ---- O += P V_j once the softmax has written P
            if (!mbar_test_wait(p_full(X), pcnt[X] & 1)) continue;
            if (nv[X] == 0 && ord[X] > 0 && !mbar_test_wait(o_free(X), (ord[X] - 1) & 1)) continue;
            const int st = pos[X] & 1;
            if (!mbar_test_wait(kv_full(X, st), (pos[X] >> 1) & 1)) continue;
            tc_fence_after();
            const uint32_t v_base = smem_u32(sKV(X, st));
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint64_t bd = smem_desc(v_base + kk * 16 * 128, BN * 128, 1024);
              umma_f16_ts(o_col, s_col + kk * 8, bd, C::IDESC_O, (nv[X] > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(kv_empty(X, st));
            ++pos[X];
            ++pcnt[X];
            ++nv[X];
            ++r[X];
            want_pv[X] = false;
            progress = true;
          }
        }
        if (progress) {
          t_last = global_timer_ns();
        } else if (*abort_flag || global_timer_ns() - t_last > kTimeoutNs) {
          ok = false;
          break;
        }
      }
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait_bounded(drain, 0, &never, kTimeoutNs);
      }
    }
  } else {
    // ================================================================ softmax
    const int X = (warp - 2) >> 2;          // slot of this warpgroup
    const int qd = warp & 3;                // TMEM lane quadrant of this warp
    const int row = qd * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const uint32_t s_col = tmem + lane_base + X * C::TM_SLOT;
    const uint32_t o_col = s_col + BN;
    int scnt = 0;
    bool ok = true;
    Item it;
    for (int ord = 0; ok && load_item(p, X, ord, it); ++ord) {
      float m_run = -INFINITY, l_run = 0.f;
      int n = 0;
      for (int r = 0; r < it.count; ++r) {
        const int j = it.list[r];
        if (j < 0 || j > it.i) continue;
        const bool diag = (j == it.i);
        if (!mbar_wait_bounded(s_full(X), scnt & 1, abort_flag, kTimeoutNs)) ok = false;
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        ++scnt;
        tc_fence_after();
        // pass 1: row maximum over the S tile (64 columns at a time)
        float mx = -INFINITY;
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float a[32], b[32];
          tmem_ld32(s_col + c0, a);
          tmem_ld32(s_col + c0 + 32, b);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float va = (diag && c0 + c > row) ? -INFINITY : a[c];
            const float vb = (diag && c0 + 32 + c > row) ? -INFINITY : b[c];
            mx = fmaxf(mx, fmaxf(va, vb));
          }
        }
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        if (n == 0) {
          m_run = m_new;
        } else if (__any_sync(0xFFFFFFFFu, m_new > m_run + kRescaleLog2)) {
          // O holds PV(0..n-1), complete: the commit that announced S(n)
          // covers every earlier MMA of this slot
          const float alpha = ex2_approx(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tmem_ld32(o_col + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= alpha;
            tmem_st32(o_col + c0, o);
          }
        }
        // pass 2: P = exp2(S * scale - m) in bf16, written over the first half
        // of the S columns (step c0 reads S[c0, c0+64) and writes P to
        // [c0/2, c0/2+32), columns whose S values were already read)
        float lsum = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float a[32], b[32];
          tmem_ld32(s_col + c0, a);
          tmem_ld32(s_col + c0 + 32, b);
          tmem_wait_ld();
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float p0 = ex2_approx(fmaf(a[c], p.scale_log2, -m_run));
            float p1 = ex2_approx(fmaf(a[c + 1], p.scale_log2, -m_run));
            if (diag && c0 + c > row) p0 = 0.f;
            if (diag && c0 + c + 1 > row) p1 = 0.f;
            lsum += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float p0 = ex2_approx(fmaf(b[c], p.scale_log2, -m_run));
            float p1 = ex2_approx(fmaf(b[c + 1], p.scale_log2, -m_run));
            if (diag && c0 + 32 + c > row) p0 = 0.f;
            if (diag && c0 + 32 + c + 1 > row) p1 = 0.f;
            lsum += p0 + p1;
            pk[16 + (c >> 1)] = pack_bf16x2(p0, p1);
          }
          tmem_st32u(s_col + (c0 >> 1), pk);
        }
        l_run += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(X));
        ++n;
      }
      if (!ok) break;
      if (!mbar_wait_bounded(o_full(X), ord & 1, abort_flag, kTimeoutNs)) ok = false;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int t = it.i * BM + row;
      const bool store = t < p.n;
      const float inv_l = (n > 0 && l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + ((size_t)it.h * p.n + t) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        if (n > 0) {
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
      mbar_arrive(o_free(X));
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
  using C = PP<D>;
  PPParams p{};
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
  p.total = a.hq * p.nb;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.status = a.status;
  auto kern = attend_pp_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SBSA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return SBSA_ERR_CUDA;
  // each CTA keeps two items in flight
  int grid = (p.total + 1) / 2;
  if (grid > sms) grid = sms;
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SBSA_OK : SBSA_ERR_CUDA;
}

}  // namespace

int launch_attend_pingpong(const AttendArgs& a, cudaStream_t stream) {
  if (a.dtype != SBSA_BF16 || a.block != 128) return SBSA_ERR_UNSUPPORTED;
  if (a.d == 128) return launch_d<128>(a, stream);
  if (a.d == 64) return launch_d<64>(a, stream);
  return SBSA_ERR_UNSUPPORTED;
}

}  // namespace sbsa
