// Attention over the selected key blocks of each query block, on the
// tcgen05 tensor cores with operands staged by TMA and accumulators in TMEM.
//
// "RBS-Attention" (iaonda.com), method paragraph: the sparse prefill stays
// compatible with sparse FlashAttention, i.e. exact softmax attention
// restricted to the kept blocks.  "MiniMax presenta MSA", "Que es MSA y como
// funciona?": the main branch runs full attention on the preselected blocks
// only.  Causal masking applies inside the diagonal block; every listed block
// j < i lies entirely before the query block.
//
// One CTA per (query head, query block), 6 warps:
//   warp 0     TMA producer: Q tile once, then K_j and V_j tiles of every
//              listed block into a 3-slot ring (128-byte swizzled boxes).
//   warp 1     TMEM owner and single-thread MMA issuer: S = Q K_j^T into a
//              double-buffered TMEM tile, O += P V_j into the TMEM output.
//   warps 2-5  one query row per thread: S row from TMEM, online softmax in
//              the exp2 domain (the running maximum is only moved, and O
//              rescaled in TMEM, when it grows by more than 2^8), P written to
//              a double-buffered shared tile in the K-major swizzled layout
//              the MMA reads, final O / l written to global memory.
// Every mbarrier wait is bounded; on expiry the CTA records SBSA_ERR_TIMEOUT,
// stops issuing work, drains its in-flight copies and MMAs and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"
#include "tma_map.h"

namespace sbsa {
namespace {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.0f;

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int size = 2;
  static constexpr uint32_t fmt = 1;  // bf16
  static constexpr CUtensorMapDataType tma = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};
template <>
struct Elem<float> {
  static constexpr int size = 4;
  static constexpr uint32_t fmt = 2;  // tf32
  static constexpr CUtensorMapDataType tma = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
};

constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <typename T, int BM, int D>
struct Cfg {
  static constexpr int BN = BM;
  static constexpr int ES = Elem<T>::size;
  static constexpr int AE = 128 / ES;   // elements in one 128-byte swizzle row
  static constexpr int NA_D = D / AE;   // swizzle atoms across d
  static constexpr int KSTEP = 32 / ES; // K of one MMA instruction
  static constexpr int Q_BYTES = BM * D * ES;
  static constexpr int KV_BYTES = BN * D * ES;
  static constexpr int P_BYTES = BM * BN * ES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_P = OFF_KV + kStages * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int NBARS = 1 + 2 * kStages + 6 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_USED = OFF_MISC + 16 + 1024;  // + base alignment slack
  // Pad so that no more CTAs share an SM than its 512 TMEM columns can hold
  // at once (a CTA whose allocation would wait only idles the SM).
  static constexpr int TM_COLS_ = pow2_at_least(2 * BN + D);
  static constexpr int SMEM_FLOOR = 233472 / (512 / TM_COLS_ + 1) + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > SMEM_FLOOR ? SMEM_USED : SMEM_FLOOR;
  // V is read MN-major: 16-bit types use the 128-byte swizzle of 16-byte
  // chunks (8-row period), 32-bit types the 128-byte swizzle of 32-byte
  // chunks (4-row period), the only MN-major layout tf32 operands accept.
  static constexpr uint32_t V_LAYOUT = ES == 4 ? kSwizzle128B_32BAtom : kSwizzle128B;
  static constexpr uint32_t V_SBO = ES == 4 ? 512 : 1024;
  static constexpr int TM_S = 0;
  static constexpr int TM_O = 2 * BN;
  static constexpr int TM_COLS = pow2_at_least(2 * BN + D);
  static constexpr uint32_t IDESC_S = make_idesc(Elem<T>::fmt, BM, BN, false, false);
  static constexpr uint32_t IDESC_O = make_idesc(Elem<T>::fmt, BM, D, false, true);
  static_assert(D % AE == 0 && BN % AE == 0, "tile widths are whole swizzle atoms");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(TM_COLS <= 512, "TMEM budget");
};

struct AttParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void* o;
  const int32_t* idx;
  const int32_t* cnt;
  int hq, n, nb, group, group_shared, kmax;
  float scale_log2;
  int* status;
};

__device__ __forceinline__ void record(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T, int BM, int D>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(const __grid_constant__ AttParams p) {
  using C = Cfg<T, BM, D>;
  constexpr int BN = C::BN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sKV = smem + C::OFF_KV;
  unsigned char* sP = smem + C::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x;
  const int i = p.nb - 1 - item / p.hq;  // longest lists first
  const int h = item % p.hq;
  const int g = h / p.group;
  const int hs = p.group_shared ? g : h;
  const int32_t* list = p.idx + ((size_t)hs * p.nb + i) * p.kmax;
  int count = p.cnt[(size_t)hs * p.nb + i];
  count = count < 0 ? 0 : (count > p.kmax ? p.kmax : count);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&pv_done[b], 1);
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
      for (int a = 0; a < C::NA_D; ++a)
        tma_load_3d(sQ + a * (BM * 128), &p.tm_q, bar_q, a * C::AE, i * BM, h);
      int issued = 0;
      bool ok = true;
      for (int r = 0; r < count && ok; ++r) {
        const int j = list[r];
        if (j < 0 || j > i) {
          record(p.status, SBSA_ERR_DEVICE);
          continue;
        }
        for (int half = 0; half < 2; ++half) {
          const int pos = issued;
          const int slot = pos % kStages;
          if (!mbar_wait_bounded(&kv_empty[slot], ((pos / kStages) & 1) ^ 1, abort_flag,
                                 kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[slot], C::KV_BYTES);
          const CUtensorMap* m = half ? &p.tm_v : &p.tm_k;
          unsigned char* dst = sKV + slot * C::KV_BYTES;
          for (int a = 0; a < C::NA_D; ++a)
            tma_load_3d(dst + a * (BN * 128), m, &kv_full[slot], a * C::AE, j * BN, g);
          ++issued;
        }
      }
      const int first = issued > kStages ? issued - kStages : 0;
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        // drain copies still landing in shared memory before the CTA exits
        volatile int never = 0;
        mbar_wait_bounded(bar_q, 0, &never, kWaitTimeoutNs);
        for (int pos = first; pos < issued; ++pos)
          mbar_wait_bounded(&kv_full[pos % kStages], (pos / kStages) & 1, &never, kWaitTimeoutNs);
      } else {
        // the MMA thread releases each slot with an asynchronous commit;
        // wait for the last release of every slot so none lands after exit
        for (int pos = first; pos < issued; ++pos)
          if (!mbar_wait_bounded(&kv_empty[pos % kStages], (pos / kStages) & 1, abort_flag,
                                 kWaitTimeoutNs))
            break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar_q, 0, abort_flag, kWaitTimeoutNs);
      tc_fence_after();
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      const uint32_t p_base = smem_u32(sP);
      int n = 0;
      auto issue_pv = [&](int m) -> bool {
        if (!mbar_wait_bounded(&p_full[m & 1], (m >> 1) & 1, abort_flag, kWaitTimeoutNs))
          return false;
        const int vpos = 2 * m + 1;
        const int slot = vpos % kStages;
        if (!mbar_wait_bounded(&kv_full[slot], (vpos / kStages) & 1, abort_flag, kWaitTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t a0 = p_base + (m & 1) * C::P_BYTES;
        const uint32_t b0 = kv_base + slot * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / C::KSTEP; ++kk) {
          const int kb = kk * 32;  // byte offset along keys in the P rows
          const uint64_t ad = smem_desc(a0 + (kb / 128) * (BM * 128) + (kb % 128), 16, 1024);
          const uint64_t bd = smem_desc(b0 + kk * C::KSTEP * 128, BN * 128, C::V_SBO, C::V_LAYOUT);
          if constexpr (C::ES == 2)
            umma_f16_ss(tmem + C::TM_O, ad, bd, C::IDESC_O, (m > 0 || kk > 0) ? 1u : 0u);
          else
            umma_tf32_ss(tmem + C::TM_O, ad, bd, C::IDESC_O, (m > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[slot]);
        umma_commit(&pv_done[m & 1]);
        return true;
      };
      for (int r = 0; r < count && ok; ++r) {
        const int j = list[r];
        if (j < 0 || j > i) continue;
        const int kpos = 2 * n;
        const int slot = kpos % kStages;
        if (!mbar_wait_bounded(&kv_full[slot], (kpos / kStages) & 1, abort_flag, kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t b0 = kv_base + slot * C::KV_BYTES;
        const uint32_t sbuf = tmem + C::TM_S + (n & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < D / C::KSTEP; ++kk) {
          const int kb = kk * 32;  // byte offset along d
          const uint64_t ad = smem_desc(q_base + (kb / 128) * (BM * 128) + (kb % 128), 16, 1024);
          const uint64_t bd = smem_desc(b0 + (kb / 128) * (BN * 128) + (kb % 128), 16, 1024);
          if constexpr (C::ES == 2)
            umma_f16_ss(sbuf, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
          else
            umma_tf32_ss(sbuf, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[n & 1]);
        umma_commit(&kv_empty[slot]);
        if (n >= 1 && !issue_pv(n - 1)) {
          ok = false;
          break;
        }
        ++n;
      }
      if (ok && n >= 1) ok = issue_pv(n - 1);
      if (!ok) {
        if (!*abort_flag) fail(SBSA_ERR_TIMEOUT);
        // wait for every MMA already issued before TMEM is released
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait_bounded(drain, 0, &never, kWaitTimeoutNs);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int qd = warp & 3;  // TMEM lane quadrant this warp may access
    const bool full_m = (BM == 128);
    const int row = full_m ? qd * 32 + lane : qd * 16 + lane;
    const bool has_row = full_m || lane < 16;
    const int t = i * BM + row;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    int n = 0;
    bool ok = true;
    for (int r = 0; r < count && ok; ++r) {
      const int j = list[r];
      if (j < 0 || j > i) continue;
      const bool diag = (j == i);
      if (!mbar_wait_bounded(&s_full[n & 1], (n >> 1) & 1, abort_flag, kWaitTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[BN];
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float chunk[32];
        tmem_ld32(tmem + lane_base + C::TM_S + (n & 1) * BN + c0, chunk);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c0 + c] = chunk[c];
      }
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        float v = has_row ? x[c] * p.scale_log2 : 0.f;
        if (diag && c > row) v = -INFINITY;
        x[c] = v;
        mx = fmaxf(mx, v);
      }
      const float m_new = fmaxf(m_run, mx);
      if (n == 0) {
        m_run = m_new;
      } else {
        const bool need = m_new > m_run + kRescaleLog2;
        if (__any_sync(0xFFFFFFFFu, need)) {
          const float alpha = ex2_approx(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
          if (!mbar_wait_bounded(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag,
                                 kWaitTimeoutNs)) {
            ok = false;
          }
          if (!__all_sync(0xFFFFFFFFu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + C::TM_O + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= alpha;
            tmem_st32(tmem + lane_base + C::TM_O + c0, o);
          }
          tmem_wait_st();
        }
      }
      // shared P buffer (n & 1) is free once PV(n - 2) has completed
      if (n >= 2) {
        if (!mbar_wait_bounded(&pv_done[n & 1], ((n - 2) >> 1) & 1, abort_flag, kWaitTimeoutNs))
          ok = false;
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
      }
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const float pv = ex2_approx(x[c] - m_run);
        x[c] = pv;
        lsum += pv;
      }
      l_run += lsum;
      if (has_row) {
        unsigned char* prow = sP + (n & 1) * C::P_BYTES + row * 128;
        const int sw = row & 7;
        if constexpr (C::ES == 2) {
#pragma unroll
          for (int ch = 0; ch < BN / 8; ++ch) {
            uint4 v;
            v.x = pack_bf16x2(x[ch * 8 + 0], x[ch * 8 + 1]);
            v.y = pack_bf16x2(x[ch * 8 + 2], x[ch * 8 + 3]);
            v.z = pack_bf16x2(x[ch * 8 + 4], x[ch * 8 + 5]);
            v.w = pack_bf16x2(x[ch * 8 + 6], x[ch * 8 + 7]);
            const int atom = ch >> 3, c16 = ch & 7;
            *reinterpret_cast<uint4*>(prow + atom * (BM * 128) + ((c16 ^ sw) << 4)) = v;
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < BN / 4; ++ch) {
            uint4 v;
            v.x = __float_as_uint(x[ch * 4 + 0]);
            v.y = __float_as_uint(x[ch * 4 + 1]);
            v.z = __float_as_uint(x[ch * 4 + 2]);
            v.w = __float_as_uint(x[ch * 4 + 3]);
            const int atom = ch >> 3, c16 = ch & 7;
            *reinterpret_cast<uint4*>(prow + atom * (BM * 128) + ((c16 ^ sw) << 4)) = v;
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[n & 1]);
      ++n;
    }
    if (ok && n > 0) {
      if (!mbar_wait_bounded(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag,
                             kWaitTimeoutNs))
        ok = false;
      // the PV before the last one signals the other barrier; consume it too
      if (ok && n > 1 &&
          !mbar_wait_bounded(&pv_done[(n - 2) & 1], ((n - 2) >> 1) & 1, abort_flag,
                             kWaitTimeoutNs))
        ok = false;
    }
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (!ok) {
      if (lane == 0 && !*abort_flag) fail(SBSA_ERR_TIMEOUT);
    } else {
      tc_fence_after();
      const float inv_l = (n > 0 && l_run > 0.f) ? 1.f / l_run : 0.f;
      T* orow = static_cast<T*>(p.o) + ((size_t)h * p.n + t) * D;
      const bool store = has_row && t < p.n;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_base + C::TM_O + c0, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0.f;
        }
        if (store) {
          if constexpr (C::ES == 2) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = pack_bf16x2(o[c + 0] * inv_l, o[c + 1] * inv_l);
              v.y = pack_bf16x2(o[c + 2] * inv_l, o[c + 3] * inv_l);
              v.z = pack_bf16x2(o[c + 4] * inv_l, o[c + 5] * inv_l);
              v.w = pack_bf16x2(o[c + 6] * inv_l, o[c + 7] * inv_l);
              *reinterpret_cast<uint4*>(orow + c0 + c) = v;
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              float4 v = make_float4(o[c] * inv_l, o[c + 1] * inv_l, o[c + 2] * inv_l,
                                     o[c + 3] * inv_l);
              *reinterpret_cast<float4*>(orow + c0 + c) = v;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

template <typename T, int BM, int D>
int launch_typed(const AttendArgs& a, cudaStream_t stream) {
  using C = Cfg<T, BM, D>;
  AttParams p{};
  const CUtensorMapDataType dt = Elem<T>::tma;
  if (!make_map(&p.tm_q, dt, C::ES, a.q, a.hq, a.n, D, BM) ||
      !make_map(&p.tm_k, dt, C::ES, a.k, a.hkv, a.n, D, BM) ||
      !make_map(&p.tm_v, dt, C::ES, a.v, a.hkv, a.n, D, BM,
                C::ES == 4 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B))
    return SBSA_ERR_CUDA;
  p.o = a.o;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.hq = a.hq;
  p.n = a.n;
  p.nb = (a.n + BM - 1) / BM;
  p.group = a.hq / a.hkv;
  p.group_shared = a.group_shared;
  p.kmax = a.kmax;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.status = a.status;
  auto kern = attend_kernel<T, BM, D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SBSA_ERR_CUDA;
  const long long grid = (long long)a.hq * p.nb;
  if (grid <= 0 || grid > 0x7FFFFFFFLL) return SBSA_ERR_INVALID_ARG;
  kern<<<(unsigned)grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SBSA_OK : SBSA_ERR_CUDA;
}

__global__ void wait_probe_kernel(uint64_t timeout_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing arrives on `bar`: the phase never completes
    if (!mbar_wait_bounded(&bar, 0, &abort_flag, timeout_ns)) record(status, SBSA_ERR_TIMEOUT);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_probe(uint64_t timeout_ns, int* status, cudaStream_t stream) {
  wait_probe_kernel<<<1, 32, 0, stream>>>(timeout_ns, status);
  return cudaGetLastError();
}

int launch_attend(const AttendArgs& a, cudaStream_t stream) {
  // 0: automatic, 1: pair, 2: persistent, 3: single, 4: duo
  static const int forced = [] {
    const char* e = std::getenv("SBSA_ATTEND_KERNEL");
    if (!e) return 0;
    if (std::strcmp(e, "pair") == 0) return 1;
    if (std::strcmp(e, "persistent") == 0) return 2;
    if (std::strcmp(e, "single") == 0) return 3;
    if (std::strcmp(e, "duo") == 0) return 4;
    return 0;
  }();
  // bf16 with 64-token blocks: the persistent kernel on two-block tiles
  if (a.dtype == SBSA_BF16 && a.block == 64 && forced != 3 && forced != 4)
    return launch_attend_persistent64(a, stream);
  const bool big = a.dtype == SBSA_BF16 && a.block == 128 && (a.d == 128 || a.d == 64);
  // The pair kernel pays off when the two heads' lists coincide (one list
  // per GQA group).  The two-tile kernel (duo) is built and tested but not
  // chosen: measured slower than the persistent kernel on per-head lists.
  const bool pairable = big && a.group_shared && (a.hq / a.hkv) % 2 == 0;
  if (forced == 3 || !big) return launch_attend_single(a, stream);
  if (forced == 4 && !a.group_shared) return launch_attend_duo(a, stream);
  if (forced == 2 || !pairable) return launch_attend_persistent(a, stream);
  return launch_attend_pair(a, stream);
}

int launch_attend_single(const AttendArgs& a, cudaStream_t stream) {
  if (a.dtype == SBSA_BF16) {
    if (a.block == 128 && a.d == 128) return launch_typed<__nv_bfloat16, 128, 128>(a, stream);
    if (a.block == 128 && a.d == 64) return launch_typed<__nv_bfloat16, 128, 64>(a, stream);
    if (a.block == 64 && a.d == 128) return launch_typed<__nv_bfloat16, 64, 128>(a, stream);
    if (a.block == 64 && a.d == 64) return launch_typed<__nv_bfloat16, 64, 64>(a, stream);
    return SBSA_ERR_UNSUPPORTED;
  }
  if (a.block == 64 && a.d == 64) return launch_typed<float, 64, 64>(a, stream);
  return SBSA_ERR_UNSUPPORTED;
}

}  // namespace sbsa
