// attn_common.cuh -- pieces shared by the attention kernels: work-unit to
// tile mapping, bounded mbarrier waits, the online-softmax step of one score
// row and the output store.
//
// The softmax follows the definition of "Core 注意力" (WorldFoundry docs,
// example section: a bool mask keeps scores, a float mask is added to them)
// and "MLA Prefill" (CANN ATB docs, parameter table: qkScale multiplies
// Q*K^T); it is evaluated online in the log2 domain:
//   x_j = s_j * qkScale * log2(e) (+ mask_j * log2(e)),  masked x_j = -inf,
//   m   = running max,  p_j = 2^(x_j - m),  l = running sum of p,
//   out = (sum_j p_j v_j) / l.
// The running max is only raised when a row's new max exceeds it by more
// than 2^8 ("lazy rescale"); p_j then stays below 2^8 and the final division
// by l cancels the stale max exactly.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "attn_params.h"
#include "sm100_ptx.cuh"

namespace wf {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units


struct TileInfo {
  int32_t b, h, hk, q0, lq, lk, qrow, krow, n_kv, off;
  int32_t tma_b, kb;   // batch coordinate of the Q / the K and V maps
  int32_t sp, kt0;     // split index, first KV tile of the split (0 without split)
};

// Sub-tile `sub` (128 rows each) of work item `t`; the enumeration order is
// described in attn_params.h (per sequence, per kv head, longest unit first,
// GQA heads adjacent; with split-KV the splits of one unit are adjacent).
// krow / n_kv describe the KV tiles this item visits: tiles [kt0, kt0 + n_kv)
// of the sequence, krow being the TMA row of tile kt0.
__device__ __forceinline__ TileInfo tile_info(const AttnParams &p, int32_t t, int32_t sub) {
  TileInfo ti;
  ti.sp = 0;
  ti.kt0 = 0;
  if (p.n_split > 1) {
    ti.sp = t % p.n_split;
    t /= p.n_split;
  }
  const int32_t G = p.group;
  const bool causal = p.mask_kind == kMaskCausal;
  int32_t r, n_units;
  if (!p.varlen) {
    n_units = p.units_per_bh;
    const int32_t per_bhk = n_units * G;                // items of one (batch, kv head)
    const int32_t blk = t / per_bhk;
    r = t - blk * per_bhk;
    ti.b = blk / p.hkv;
    ti.hk = blk - ti.b * p.hkv;
    ti.lq = p.lq;
    ti.lk = p.lk;
    ti.krow = 0;
    ti.tma_b = ti.b;
    ti.kb = ti.b;
  } else {
    const int32_t *cu_work = p.ws + p.sl.cu_work;
    int32_t lo = 0, hi = p.batch - 1;                   // last k with cu_work[k] <= t
    while (lo < hi) {
      const int32_t mid = (lo + hi + 1) >> 1;
      if (__ldg(cu_work + mid) <= t) lo = mid; else hi = mid - 1;
    }
    ti.b = __ldg(p.ws + p.sl.order + lo);
    r = t - __ldg(cu_work + lo);
    const int32_t cq = __ldg(p.ws + p.sl.cu_q + ti.b), ck = __ldg(p.ws + p.sl.cu_k + ti.b);
    ti.lq = __ldg(p.ws + p.sl.cu_q + ti.b + 1) - cq;
    ti.lk = __ldg(p.ws + p.sl.cu_k + ti.b + 1) - ck;
    ti.krow = p.kv_padded ? 0 : ck;      // padded: sequence b's keys start row 0 of batch b
    ti.tma_b = 0;
    ti.kb = p.kv_padded ? ti.b : 0;
    n_units = (ti.lq + p.unit_rows - 1) / p.unit_rows;
    ti.hk = r / (n_units * G);
    r -= ti.hk * n_units * G;
  }
  const int32_t j = r / G;
  ti.h = ti.hk * G + (r - j * G);
  const int32_t u = causal ? n_units - 1 - j : j;
  const int32_t u0 = u * p.unit_rows;
  ti.q0 = u0 + sub * kBlockM;
  ti.qrow = (p.varlen ? __ldg(p.ws + p.sl.cu_q + ti.b) : 0) + ti.q0;
  ti.off = p.causal_top_left ? 0 : ti.lk - ti.lq;   // causal: last visible key of row i is i + off
  int32_t kend = ti.q0 < ti.lq ? ti.lk : 0;            // no valid row: nothing to do
  if (causal) {
    const int32_t last = min(ti.q0 + kBlockM, ti.lq);   // one past the last valid row
    kend = min(kend, last + ti.off);
  }
  ti.n_kv = kend > 0 ? (kend + kBlockN - 1) / kBlockN : 0;
  if (p.n_split > 1) {
    // The split bounds come from the whole unit, so both sub-tiles of a unit
    // visit the same KV tiles (the CTA loads each tile once for both).
    int32_t uend = u0 < ti.lq ? ti.lk : 0;
    if (causal) uend = min(uend, min(u0 + p.unit_rows, ti.lq) + ti.off);
    const int32_t n_unit = uend > 0 ? (uend + kBlockN - 1) / kBlockN : 0;
    const int32_t per = (n_unit + p.n_split - 1) / p.n_split;
    const int32_t lo = min(ti.sp * per, n_unit);
    ti.kt0 = lo;
    ti.n_kv = max(min(lo + per, ti.n_kv) - lo, 0);
    ti.krow += lo * kBlockN;
  }
  return ti;
}

__device__ __forceinline__ int32_t num_units(const AttnParams &p) {
  const int32_t base = p.varlen ? __ldg(p.ws) : p.n_units_dense;
  return p.n_split > 1 ? base * p.n_split : base;
}

// Bounded wait.  Returns false (and raises the CTA abort flag) on expiry, or
// if another role already aborted.
__device__ __forceinline__ bool bwait(uint64_t *bar, uint32_t parity, volatile int32_t *abort,
                                      const AttnParams &p) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > p.timeout_cycles) {
      *abort = 1;
      atomicCAS(p.status, 0, kDevTimeout);
      return false;
    }
  }
}

// Wait used while draining after an abort: ignores the abort flag, still bounded.
__device__ __forceinline__ bool drain_wait(uint64_t *bar, uint32_t parity, const AttnParams &p) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > p.timeout_cycles) {
      atomicCAS(p.status, 0, kDevTimeout);
      return false;
    }
  }
  return true;
}

// Last fill index the producer issued per barrier (-1: none), for the drain.
struct ProducerLog {
  int32_t q_last;
  int32_t k_last[3], v_last[3];
};

// One softmax step of one score row (128 keys starting at k0).  `sr` holds the
// raw fp32 scores; on return `x` holds p_j (0 for masked keys), m / l are
// updated, and the return value is the factor O must be multiplied by
// (1 when the running max did not move).
// kEmuPer16: of every 16 score columns, this many are exponentiated on the FMA
// pipe (exp2_poly2) instead of the MUFU unit, in tiles without masked scores.
// At head size 128 the MUFU rate alone (16 per clock per SM) makes one
// tile's softmax as long as the other tile's two MMAs.
// kExplicit: the instance that reads explicit masks (p.mask_kind keep or
// add); without it only no mask and the causal mask are handled.
// kPSplit > 0: `mid(alpha)` is called once p_0 .. p_{kPSplit-1} are final,
// before the remaining columns are exponentiated (the caller hands that part
// of P to the PV product early).
template <int C0, int C1, int kEmuPer16>
__device__ __forceinline__ void exp_cols(float (&x)[128], float (&sq)[8], float sc, float neg_m) {
#pragma unroll
  for (int c = C0; c < C1; c += 2) {
    fma2_bc(x[c], x[c + 1], x[c], x[c + 1], sc, neg_m);
    if ((c & 15) < kEmuPer16) {
      exp2_poly2(x[c], x[c + 1]);
    } else {
      x[c] = ex2_approx(x[c]);
      x[c + 1] = ex2_approx(x[c + 1]);
    }
    const int q = (c >> 1) & 3;
    add2(sq[2 * q], sq[2 * q + 1], x[c], x[c + 1]);
  }
}

template <int kEmuPer16, bool kExplicit, int kPSplit = 0, typename Mid>
__device__ __forceinline__ float softmax_row(const AttnParams &p, const TileInfo &ti, int32_t row,
                                             int32_t k0, const uint32_t (&sr)[128],
                                             float (&x)[128], float &m, float &l, Mid &&mid) {
  const bool causal = p.mask_kind == kMaskCausal;
  const bool explicit_mask = kExplicit && (p.mask_kind == kMaskKeep || p.mask_kind == kMaskAdd);
  const bool row_valid = row < ti.lq;
  int32_t lim = ti.lk - 1 - k0;                      // last visible column of this row
  if (causal) lim = min(lim, row + ti.off - k0);
  const bool need_mask = (k0 + kBlockN > ti.lk) || (causal && (k0 + kBlockN - 1 > ti.q0 + ti.off));
  // prescaled: x holds scaled scores after the first pass (explicit masks, or a
  // non-positive scale for which max and scaling do not commute)
  const bool prescaled = explicit_mask || !(p.scale_log2 > 0.f);
  // pass 1: x = (masked) scores, and their max in four independent chains of
  // three-input max.
  if (!prescaled) {
    if (need_mask) {
#pragma unroll
      for (int c = 0; c < 128; ++c) x[c] = (c <= lim) ? __uint_as_float(sr[c]) : -INFINITY;
    } else {
#pragma unroll
      for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c]);
    }
  } else if (!explicit_mask) {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      x[c] = (c <= lim) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
  } else if constexpr (kExplicit) {
    const int64_t mrow = (int64_t)ti.b * p.m_sb + (int64_t)ti.h * p.m_sh + (int64_t)row * p.m_si;
    // A full tile of a mask whose keys are contiguous and 16-byte aligned is
    // read with 16-byte loads: a thread's 128 entries in a few vector loads
    // instead of 128 scattered element loads.
    const int es = p.mask_kind == kMaskKeep ? 1 : (p.mask_dtype == kMaskF32 ? 4 : 2);
    const uint8_t *mrow_k0 = reinterpret_cast<const uint8_t *>(p.mask) + (mrow + k0) * es;
    const bool vec = p.m_sj == 1 && k0 + kBlockN <= ti.lk &&
                     (reinterpret_cast<uintptr_t>(mrow_k0) & 15) == 0;
    if (p.mask_kind == kMaskKeep && vec) {
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = row_valid ? __ldg(reinterpret_cast<const uint4 *>(mrow_k0) + i) : make_uint4(0, 0, 0, 0);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const bool keep = c <= lim && ((w[c >> 2] >> (8 * (c & 3))) & 0xffu) != 0u;
        x[c] = keep ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
      }
    } else if (p.mask_kind == kMaskKeep) {
      const uint8_t *mp = reinterpret_cast<const uint8_t *>(p.mask) + mrow;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const bool keep = row_valid && c <= lim && mp[(int64_t)(k0 + c) * p.m_sj] != 0;
        x[c] = keep ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
      }
    } else if (vec) {
      // additive, 16 entries at a time (one or two 16-byte loads per 8)
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 16) {
        float a[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint8_t *src = mrow_k0 + (int64_t)(c0 + 8 * h) * es;
          if (p.mask_dtype == kMaskF32) {
            const float4 u = row_valid ? __ldg(reinterpret_cast<const float4 *>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 v = row_valid ? __ldg(reinterpret_cast<const float4 *>(src) + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
            a[8 * h + 0] = u.x; a[8 * h + 1] = u.y; a[8 * h + 2] = u.z; a[8 * h + 3] = u.w;
            a[8 * h + 4] = v.x; a[8 * h + 5] = v.y; a[8 * h + 6] = v.z; a[8 * h + 7] = v.w;
          } else {
            const uint4 u = row_valid ? __ldg(reinterpret_cast<const uint4 *>(src)) : make_uint4(0, 0, 0, 0);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float2 f;
              if (p.mask_dtype == kMaskBF16)
                f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&uw[i]));
              else
                f = __half22float2(*reinterpret_cast<const __half2 *>(&uw[i]));
              a[8 * h + 2 * i] = f.x;
              a[8 * h + 2 * i + 1] = f.y;
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const bool in = row_valid && c0 + c <= lim;
          x[c0 + c] = in ? fmaf(a[c], kLog2e, __uint_as_float(sr[c0 + c]) * p.scale_log2) : -INFINITY;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float add = 0.f;
        const bool in = row_valid && c <= lim;
        if (in) {
          const int64_t idx = mrow + (int64_t)(k0 + c) * p.m_sj;
          add = p.mask_dtype == kMaskF32
                    ? reinterpret_cast<const float *>(p.mask)[idx]
                    : p.mask_dtype == kMaskBF16
                          ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p.mask)[idx])
                          : __half2float(reinterpret_cast<const __half *>(p.mask)[idx]);
        }
        x[c] = in ? fmaf(add, kLog2e, __uint_as_float(sr[c]) * p.scale_log2) : -INFINITY;
      }
    }
  }
  float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < 128; c += 8) {
#pragma unroll
    for (int q = 0; q < 4; ++q) mq[q] = fmax3(mq[q], x[c + 2 * q], x[c + 2 * q + 1]);
  }
  float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
  if (!prescaled) mx *= p.scale_log2;                // -inf stays -inf (scale > 0)
  const float m_new = fmaxf(m, mx);
  float alpha = 1.f;
  if (m == -INFINITY) {
    m = m_new;                                       // nothing accumulated yet
  } else if (m_new > m + kRescaleThreshold) {
    alpha = ex2_approx(m - m_new);
    m = m_new;
  }
  // pass 2: p = 2^(x * sc - m) (packed FMA), row sum in four packed partial sums
  const float neg_m = (m == -INFINITY) ? 0.f : -m;
  const float sc = prescaled ? 1.f : p.scale_log2;
  float sq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (kEmuPer16 > 0 && !prescaled && !need_mask) {
    exp_cols<0, kPSplit, kEmuPer16>(x, sq, sc, neg_m);
    if constexpr (kPSplit > 0) mid(alpha);
    exp_cols<kPSplit, 128, kEmuPer16>(x, sq, sc, neg_m);
  } else {
    exp_cols<0, kPSplit, 0>(x, sq, sc, neg_m);
    if constexpr (kPSplit > 0) mid(alpha);
    exp_cols<kPSplit, 128, 0>(x, sq, sc, neg_m);
  }
  const float sum = ((sq[0] + sq[1]) + (sq[2] + sq[3])) + ((sq[4] + sq[5]) + (sq[6] + sq[7]));
  l = l * alpha + sum;
  return alpha;
}

// Normalised output row (DV values) to global memory; 16-byte stores.
template <typename T, int DV>
__device__ __forceinline__ void store_row(const AttnParams &p, const TileInfo &ti, int32_t row,
                                          const float (&o)[DV], float inv) {
  T *dst = reinterpret_cast<T *>(p.out) + (int64_t)ti.b * p.o_sb + (int64_t)ti.h * p.o_sh +
           (int64_t)(p.varlen ? ti.qrow + (row - ti.q0) : row) * p.o_si;
  // One thread writes one row, so every store instruction of a warp touches
  // 32 rows; 32-byte stores halve the instructions and the cache-line visits
  // against 16-byte ones (rows whose start is not 32-byte aligned take those).
  if constexpr (sizeof(T) == 2) {
    if (DV % 16 == 0 && (reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
#pragma unroll
      for (int c = 0; c < DV; c += 16) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = Elem16<T>::pack2(o[c + 2 * i] * inv, o[c + 2 * i + 1] * inv);
        st_global_v8(dst + c, w);
      }
      return;
    }
#pragma unroll
    for (int c = 0; c < DV; c += 8) {
      uint4 v;
      v.x = Elem16<T>::pack2(o[c + 0] * inv, o[c + 1] * inv);
      v.y = Elem16<T>::pack2(o[c + 2] * inv, o[c + 3] * inv);
      v.z = Elem16<T>::pack2(o[c + 4] * inv, o[c + 5] * inv);
      v.w = Elem16<T>::pack2(o[c + 6] * inv, o[c + 7] * inv);
      *reinterpret_cast<uint4 *>(dst + c) = v;
    }
  } else {
    if (DV % 8 == 0 && (reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
#pragma unroll
      for (int c = 0; c < DV; c += 8) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(o[c + i] * inv);
        st_global_v8(dst + c, w);
      }
      return;
    }
#pragma unroll
    for (int c = 0; c < DV; c += 4) {
      float4 v = make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
      *reinterpret_cast<float4 *>(dst + c) = v;
    }
  }
}

// Result of one row: O / l to out (and its LSE when asked for), or, with
// split-KV, the partial row normalised over this split's keys plus its LSE to
// the partial buffers.  LSE = ln sum_j exp(x_j) = (m + log2 l) ln 2, -inf for a
// row that saw no key (l = 0, O = 0).
template <typename T, int DV>
__device__ __forceinline__ void store_result(const AttnParams &p, const TileInfo &ti, int32_t row,
                                             const float (&o)[DV], float m, float l) {
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float lse = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
  if (p.n_split > 1) {
    const int64_t r = p.varlen ? (int64_t)(ti.qrow - ti.q0 + row) * p.hq + ti.h
                               : ((int64_t)ti.b * p.hq + ti.h) * p.lq + row;
    const int64_t idx = (int64_t)ti.sp * p.part_rows + r;
    float *dst = p.part_o + idx * DV;       // 256-byte aligned buffer, DV % 8 == 0
#pragma unroll
    for (int c = 0; c < DV; c += 8) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(o[c + i] * inv);
      st_global_v8(dst + c, w);
    }
    p.part_lse[idx] = lse;
  } else {
    store_row<T, DV>(p, ti, row, o, inv);
    if (p.lse)
      p.lse[(int64_t)ti.b * p.l_sb + (int64_t)ti.h * p.l_sh +
            (int64_t)(p.varlen ? ti.qrow + (row - ti.q0) : row) * p.l_si] = lse;
  }
}

template <typename T, int DV>
__device__ __forceinline__ void store_zero_row(const AttnParams &p, const TileInfo &ti,
                                               int32_t row) {
  float z[DV];
#pragma unroll
  for (int c = 0; c < DV; ++c) z[c] = 0.f;
  store_result<T, DV>(p, ti, row, z, -INFINITY, 0.f);
}

// Load DV fp32 columns of this thread's TMEM lane starting at `taddr`.
template <int DV>
__device__ __forceinline__ void tmem_load_row(uint32_t taddr, float (&o)[DV]) {
  if constexpr (DV == 128) {      // one load and one wait for the whole row
    uint32_t oc[128];
    tmem_ld_x128(taddr, oc);
#pragma unroll
    for (int c = 0; c < 128; ++c) o[c] = __uint_as_float(oc[c]);
  } else {
#pragma unroll
    for (int c0 = 0; c0 < DV; c0 += 32) {
      uint32_t oc[32];
      tmem_ld_x32(taddr + c0, oc);
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c0 + c] = __uint_as_float(oc[c]);
    }
  }
}

// O row *= alpha in TMEM (DV columns).
template <int DV>
__device__ __forceinline__ void tmem_scale_row(uint32_t taddr, float alpha) {
#pragma unroll
  for (int c0 = 0; c0 < DV; c0 += 32) {
    uint32_t o[32];
    tmem_ld_x32(taddr + c0, o);
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
    tmem_st_x32(taddr + c0, o);
  }
}

// P (128 values) into TMEM over the score columns: 16-bit pairs of the
// input type T (64 columns), or for T = float the fp32 bits read by the TF32
// MMA (128 columns).
template <typename T>
__device__ __forceinline__ void tmem_store_p(uint32_t taddr, const float (&x)[128]) {
  uint32_t pk[64];
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int c = 0; c < 64; ++c) pk[c] = Elem16<T>::pack2(x[2 * c], x[2 * c + 1]);
    tmem_st_x64(taddr, pk);
  } else {
#pragma unroll
    for (int c = 0; c < 64; ++c) pk[c] = __float_as_uint(x[c]);
    tmem_st_x64(taddr, pk);
#pragma unroll
    for (int c = 0; c < 64; ++c) pk[c] = __float_as_uint(x[64 + c]);
    tmem_st_x64(taddr + 64, pk);
  }
}

// P values [C0, C1) of the row (16-bit pairs) into TMEM columns C0/2 ..
// C1/2 of the score slot at `taddr`, where the PV product reads keys C0 .. C1;
// stored as 32-, 16- and 8-column pieces.
template <typename T, int C0, int C1>
__device__ __forceinline__ void tmem_store_p_part(uint32_t taddr, const float (&x)[128]) {
  static_assert(sizeof(T) == 2 && C0 % 16 == 0 && C1 % 16 == 0 && C0 <= C1 && C1 <= 128, "P part");
  constexpr int N = (C1 - C0) / 2;
  if constexpr (N > 0) {
    uint32_t pk[N];
#pragma unroll
    for (int c = 0; c < N; ++c) pk[c] = Elem16<T>::pack2(x[C0 + 2 * c], x[C0 + 2 * c + 1]);
    constexpr int n64 = N & 64, n32 = N & 32, n16 = N & 16;
    const uint32_t a = taddr + C0 / 2;
    if constexpr (n64 != 0) tmem_st_x64(a, *reinterpret_cast<const uint32_t(*)[64]>(pk));
    if constexpr (n32 != 0) tmem_st_x32(a + n64, *reinterpret_cast<const uint32_t(*)[32]>(pk + n64));
    if constexpr (n16 != 0) tmem_st_x16(a + n64 + n32, pk + n64 + n32);
    if constexpr ((N & 8) != 0) tmem_st_x8(a + n64 + n32 + n16, pk + n64 + n32 + n16);
  }
}

}  // namespace wf
