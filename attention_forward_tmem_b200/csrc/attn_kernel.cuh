// attn_kernel.cuh -- single-tile attention forward for sm_100a (used where
// two query tiles do not fit in shared memory: the fp32 / TF32 path).
//
// Computes, per query row i of head h (kv head g = h / (Hq / Hkv)):
//     out[i] = sum_j softmax_j(qkScale * (q_i . k_j + qRope_i . kRope_j) + mask_ij) v_j
// the operation of "Core 注意力" (WorldFoundry docs, section "选择最窄的入口":
// PyTorch SDPA contract with GQA) and of "MLA Prefill" (CANN ATB docs,
// parameter table).
//
// One CTA per SM, persistent over 128-row work units, 192 threads:
//   warp 4      TMA producer: Q once per unit, then K and V tiles through a
//               STAGES-deep mbarrier ring (128-byte swizzle).
//   warp 5      tcgen05 issuer (one thread): S = Q K^T into one of two TMEM
//               S buffers, then O += P V with P read from TMEM.  S for tile
//               j+1 is issued before PV for tile j, so the tensor core works
//               on the next scores while the softmax runs.
//   warps 0-3   one thread per query row: softmax_row() on the score row, P
//               written back over S, O rescaled in TMEM when the running max
//               moved, finally O / l stored.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+DV); 512 allocated.
// Every mbarrier wait is bounded (see attn_common.cuh).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "attn_common.cuh"

namespace wf {

template <typename T, int DQK, int DROPE, int DV>
struct AttnCfg {
  static constexpr int kES = sizeof(T);
  static constexpr bool kTF32 = (kES == 4);
  static constexpr int kAtomE = 128 / kES;             // elements per 128-byte row
  static constexpr int kKStep = 32 / kES;              // MMA K per instruction
  static constexpr int kQAtoms = (DQK + kAtomE - 1) / kAtomE;
  static constexpr int kRAtoms = DROPE / kAtomE;
  static constexpr int kQKAtoms = kQAtoms + kRAtoms;
  // bf16: V tile [128 keys][DV] used MN-major, DV split into 128-byte atoms.
  // TF32 (MN-major B not available): V^T tile [DV rows][128 keys] used
  // K-major, the keys split into 128-byte atoms.
  static constexpr bool kVKMajor = kTF32;
  static constexpr int kVAtoms = kVKMajor ? kBlockN / kAtomE : (DV + kAtomE - 1) / kAtomE;
  static constexpr int kAtomBytes = 128 * 128;         // 128 rows x 128 bytes
  static constexpr int kQBytes = kQKAtoms * kAtomBytes;
  static constexpr int kKBytes = kQKAtoms * kAtomBytes;
  static constexpr int kVBytes = kVAtoms * kAtomBytes;
  static constexpr int kBudget = 227 * 1024 - 2048;    // leave room for control block + align
  static constexpr int kStagesFit = (kBudget - kQBytes) / (kKBytes + kVBytes);
  static constexpr int kStages = kStagesFit > 3 ? 3 : kStagesFit;
  static constexpr int kKOff = kQBytes;
  static constexpr int kVOff = kKOff + kStages * kKBytes;
  static constexpr int kCtrlOff = kVOff + kStages * kVBytes;
  // At least 120 KB so that two CTAs never share an SM: each allocates all
  // 512 TMEM columns.
  static constexpr int kSmemUsed = kCtrlOff + 1024 /*ctrl*/ + 1024 /*align slack*/;
  static constexpr int kSmemBytes = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  static constexpr int kSKStepsQK = DQK / kKStep;
  static constexpr int kSKStepsR = DROPE / kKStep;
  static constexpr int kPVKSteps = kBlockN / kKStep;
  static constexpr uint32_t kFmt = kTF32 ? 2u : 1u;
  static constexpr uint32_t kIdescS = instr_desc(kFmt, kBlockM, kBlockN, 0);
  // PV runs over whole 128-byte V atoms (zero-filled past DV by the TMA), so
  // its N never ends inside a swizzle atom.
  static constexpr int kNPV = kVKMajor ? DV : kVAtoms * kAtomE;
  static constexpr uint32_t kIdescPV = instr_desc(kFmt, kBlockM, kNPV, kVKMajor ? 0 : 1);
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kOCol = 256;
  static_assert(kStages >= 1, "tile does not fit in shared memory");
  static_assert(DQK % kKStep == 0 && DV % 32 == 0 && DROPE % kAtomE == 0, "head dims");
  static_assert(DV <= 128 && DV >= 32 && kNPV <= 128 && kNPV % 16 == 0, "DV");
};

struct AttnCtrl {
  uint64_t q_full, q_empty, o_empty, drain;
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint32_t tmem_base;
  volatile int32_t abort;
};

// ------------------------------------------------------------------ producer
template <typename Cfg>
__device__ void producer_role(const AttnParams &p, uint8_t *smem, AttnCtrl *ctl,
                              ProducerLog &log) {
  tma_prefetch_map(&p.tm_q);
  tma_prefetch_map(&p.tm_k);
  tma_prefetch_map(&p.tm_v);
  if (Cfg::kRAtoms) {
    tma_prefetch_map(&p.tm_qr);
    tma_prefetch_map(&p.tm_kr);
  }
  const int32_t n_units = num_units(p);
  uint32_t g = 0, u = 0;
  int32_t *k_last = log.k_last, *v_last = log.v_last;
  log.q_last = -1;
  for (int i = 0; i < 3; ++i) k_last[i] = v_last[i] = -1;
  bool ok = true;
  bool starve = (p.debug_flags & kDebugStarveFirstK) != 0;
  for (int32_t t = blockIdx.x; t < n_units && ok; t += gridDim.x) {
    const TileInfo ti = tile_info(p, t, 0);
    if (ti.n_kv == 0) continue;
    if (!(ok = bwait(&ctl->q_empty, (u + 1) & 1, &ctl->abort, p))) break;
    mbar_arrive_expect_tx(&ctl->q_full, Cfg::kQBytes);
    log.q_last = static_cast<int32_t>(u);
#pragma unroll
    for (int a = 0; a < Cfg::kQAtoms; ++a)
      tma_load_4d(smem + a * Cfg::kAtomBytes, &p.tm_q, &ctl->q_full, a * Cfg::kAtomE, ti.qrow,
                  ti.h, ti.tma_b);
#pragma unroll
    for (int a = 0; a < Cfg::kRAtoms; ++a)
      tma_load_4d(smem + (Cfg::kQAtoms + a) * Cfg::kAtomBytes, &p.tm_qr, &ctl->q_full,
                  a * Cfg::kAtomE, ti.qrow, ti.h, ti.tma_b);
    for (int32_t j = 0; j < ti.n_kv; ++j) {
      const uint32_t gg = g + j, st = gg % Cfg::kStages, n = gg / Cfg::kStages;
      const int32_t krow = ti.krow + j * kBlockN;
      if (!(ok = bwait(&ctl->k_empty[st], (n + 1) & 1, &ctl->abort, p))) break;
      if (starve) {
        starve = false;     // debug: this K tile is never loaded, its consumer times out
      } else {
        uint8_t *kdst = smem + Cfg::kKOff + st * Cfg::kKBytes;
        mbar_arrive_expect_tx(&ctl->k_full[st], Cfg::kKBytes);
#pragma unroll
        for (int a = 0; a < Cfg::kQAtoms; ++a)
          tma_load_4d(kdst + a * Cfg::kAtomBytes, &p.tm_k, &ctl->k_full[st], a * Cfg::kAtomE, krow,
                      ti.hk, ti.kb);
#pragma unroll
        for (int a = 0; a < Cfg::kRAtoms; ++a)
          tma_load_4d(kdst + (Cfg::kQAtoms + a) * Cfg::kAtomBytes, &p.tm_kr, &ctl->k_full[st],
                      a * Cfg::kAtomE, krow, ti.hk, ti.kb);
        k_last[st] = static_cast<int32_t>(n);
      }
      if (!(ok = bwait(&ctl->v_empty[st], (n + 1) & 1, &ctl->abort, p))) break;
      uint8_t *vdst = smem + Cfg::kVOff + st * Cfg::kVBytes;
      mbar_arrive_expect_tx(&ctl->v_full[st], Cfg::kVBytes);
#pragma unroll
      for (int a = 0; a < Cfg::kVAtoms; ++a) {
        if constexpr (Cfg::kVKMajor)   // V^T: (keys, DV rows) box at key offset a*kAtomE
          tma_load_4d(vdst + a * Cfg::kAtomBytes, &p.tm_v, &ctl->v_full[st], krow + a * Cfg::kAtomE,
                      0, ti.hk, ti.kb);
        else
          tma_load_4d(vdst + a * Cfg::kAtomBytes, &p.tm_v, &ctl->v_full[st], a * Cfg::kAtomE, krow,
                      ti.hk, ti.kb);
      }
      v_last[st] = static_cast<int32_t>(n);
    }
    if (!ok) break;
    g += ti.n_kv;
    ++u;
  }
}

// Wait (bounded) for every copy the producer started, so that no TMA write
// can land after the CTA has released its shared memory.  Run after all roles
// finished; in a normal run every one of these phases is already complete.
template <typename Ctrl>
__device__ void producer_drain(const AttnParams &p, Ctrl *ctl, const ProducerLog &log,
                               int k_stages, int v_stages) {
  if (log.q_last >= 0) drain_wait(&ctl->q_full, log.q_last & 1, p);
  for (int s = 0; s < k_stages; ++s)
    if (log.k_last[s] >= 0) drain_wait(&ctl->k_full[s], log.k_last[s] & 1, p);
  for (int s = 0; s < v_stages; ++s)
    if (log.v_last[s] >= 0) drain_wait(&ctl->v_full[s], log.v_last[s] & 1, p);
}

// ----------------------------------------------------------------------- MMA
template <typename Cfg>
__device__ __forceinline__ void issue_pv(const AttnParams &p, uint8_t *smem, AttnCtrl *ctl,
                                         uint32_t tmem, uint32_t gg, bool first, uint32_t u,
                                         bool &ok) {
  const uint32_t st = gg % Cfg::kStages, sb = gg & 1;
  if (first && !(ok = bwait(&ctl->o_empty, (u + 1) & 1, &ctl->abort, p))) return;
  if (!(ok = bwait(&ctl->p_full[sb], (gg >> 1) & 1, &ctl->abort, p))) return;
  if (!(ok = bwait(&ctl->v_full[st], (gg / Cfg::kStages) & 1, &ctl->abort, p))) return;
  tc_fence_after();
  const uint32_t vbase = smem_u32(smem + Cfg::kVOff + st * Cfg::kVBytes);
#pragma unroll
  for (int ks = 0; ks < Cfg::kPVKSteps; ++ks) {
    const uint64_t bdesc =
        Cfg::kVKMajor ? smem_desc_sw128(vbase + (ks / 4) * Cfg::kAtomBytes + (ks % 4) * 32, 16, 1024)
                      : smem_desc_sw128(vbase + ks * Cfg::kKStep * 128, Cfg::kAtomBytes, 1024);
    const uint32_t a_tmem = tmem + sb * 128 + ks * 8;
    if constexpr (Cfg::kTF32)
      mma_tf32_ts(tmem + Cfg::kOCol, a_tmem, bdesc, Cfg::kIdescPV, (!first || ks > 0) ? 1u : 0u);
    else
      mma_f16_ts(tmem + Cfg::kOCol, a_tmem, bdesc, Cfg::kIdescPV, (!first || ks > 0) ? 1u : 0u);
  }
  tc_commit(&ctl->v_empty[st]);
  tc_commit(&ctl->pv_done[sb]);
}

template <typename Cfg>
__device__ void mma_role(const AttnParams &p, uint8_t *smem, AttnCtrl *ctl, uint32_t tmem) {
  const int32_t n_units = num_units(p);
  const uint32_t qbase = smem_u32(smem);
  uint32_t g = 0, u = 0;
  bool ok = true;
  for (int32_t t = blockIdx.x; t < n_units && ok; t += gridDim.x) {
    const TileInfo ti = tile_info(p, t, 0);
    if (ti.n_kv == 0) continue;
    if (!(ok = bwait(&ctl->q_full, u & 1, &ctl->abort, p))) break;
    tc_fence_after();
    for (int32_t j = 0; j < ti.n_kv; ++j) {
      const uint32_t gg = g + j, st = gg % Cfg::kStages, sb = gg & 1;
      if (!(ok = bwait(&ctl->k_full[st], (gg / Cfg::kStages) & 1, &ctl->abort, p))) break;
      // S buffer sb was last read (as P) by PV[gg-2]
      if (gg >= 2 && !(ok = bwait(&ctl->pv_done[sb], ((gg - 2) >> 1) & 1, &ctl->abort, p))) break;
      tc_fence_after();
      const uint32_t kbase = smem_u32(smem + Cfg::kKOff + st * Cfg::kKBytes);
#pragma unroll
      for (int ks = 0; ks < Cfg::kSKStepsQK + Cfg::kSKStepsR; ++ks) {
        const int atom = ks < Cfg::kSKStepsQK ? ks / 4 : Cfg::kQAtoms + (ks - Cfg::kSKStepsQK) / 4;
        const int within = (ks < Cfg::kSKStepsQK ? ks % 4 : (ks - Cfg::kSKStepsQK) % 4) * 32;
        const uint32_t off = atom * Cfg::kAtomBytes + within;
        const uint64_t adesc = smem_desc_sw128(qbase + off, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(kbase + off, 16, 1024);
        if constexpr (Cfg::kTF32)
          mma_tf32_ss(tmem + sb * 128, adesc, bdesc, Cfg::kIdescS, ks > 0 ? 1u : 0u);
        else
          mma_f16_ss(tmem + sb * 128, adesc, bdesc, Cfg::kIdescS, ks > 0 ? 1u : 0u);
      }
      tc_commit(&ctl->k_empty[st]);
      tc_commit(&ctl->s_full[sb]);
      if (j == ti.n_kv - 1) tc_commit(&ctl->q_empty);
      if (j > 0) {
        issue_pv<Cfg>(p, smem, ctl, tmem, gg - 1, j == 1, u, ok);
        if (!ok) break;
      }
    }
    if (!ok) break;
    issue_pv<Cfg>(p, smem, ctl, tmem, g + ti.n_kv - 1, ti.n_kv == 1, u, ok);
    if (!ok) break;
    g += ti.n_kv;
    ++u;
  }
  // Drain: every MMA this thread issued must finish before TMEM is freed
  // (after an abort some of them were never waited on).
  tc_commit(&ctl->drain);
  drain_wait(&ctl->drain, 0, p);
}

// ------------------------------------------------------------------- softmax
template <typename T, typename Cfg, int DV>
__device__ void softmax_role(const AttnParams &p, AttnCtrl *ctl, uint32_t tmem) {
  const int32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t r = threadIdx.x;                       // row within the tile = TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const int32_t n_units = num_units(p);
  uint32_t g = 0;
  bool ok = true;
  for (int32_t t = blockIdx.x; t < n_units && ok; t += gridDim.x) {
    const TileInfo ti = tile_info(p, t, 0);
    const int32_t row = ti.q0 + r;
    const bool row_valid = row < ti.lq;
    if (ti.n_kv == 0) {
      if (row_valid) store_zero_row<T, DV>(p, ti, row);
      continue;
    }
    float m = -INFINITY, l = 0.f;
    for (int32_t j = 0; j < ti.n_kv; ++j) {
      const uint32_t gg = g + j, sb = gg & 1;
      if (!(ok = bwait(&ctl->s_full[sb], (gg >> 1) & 1, &ctl->abort, p))) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128(tmem + lane_base + sb * 128, sr);
      float x[128];
      const float alpha = softmax_row<0, true>(p, ti, row, (ti.kt0 + j) * kBlockN, sr, x, m, l,
                                                 [](float) {});
      tmem_store_p<T>(tmem + lane_base + sb * 128, x);
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O holds the sum up to tile j-1 once PV[gg-1] is done.
        if (!(ok = bwait(&ctl->pv_done[(gg - 1) & 1], ((gg - 1) >> 1) & 1, &ctl->abort, p))) {
          tmem_st_wait();
          break;
        }
        tc_fence_after();
        tmem_scale_row<DV>(tmem + lane_base + Cfg::kOCol, alpha);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[sb]);
    }
    if (!ok) break;
    g += ti.n_kv;
    // Epilogue: O is final once the last PV of this tile is done.
    const uint32_t gl = g - 1;
    if (!(ok = bwait(&ctl->pv_done[gl & 1], (gl >> 1) & 1, &ctl->abort, p))) break;
    tc_fence_after();
    float o[DV];
    tmem_load_row<DV>(tmem + lane_base + Cfg::kOCol, o);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->o_empty);
    if (row_valid) store_result<T, DV>(p, ti, row, o, m, l);
  }
}

// --------------------------------------------------------------------- kernel
template <typename T, int DQK, int DROPE, int DV>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using Cfg = AttnCfg<T, DQK, DROPE, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  AttnCtrl *ctl = reinterpret_cast<AttnCtrl *>(smem + Cfg::kCtrlOff);
  const int32_t warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    mbar_init(&ctl->o_empty, 4);
    mbar_init(&ctl->drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->p_full[i], 4);
      mbar_init(&ctl->pv_done[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&ctl->k_full[i], 1);
      mbar_init(&ctl->k_empty[i], 1);
      mbar_init(&ctl->v_full[i], 1);
      mbar_init(&ctl->v_empty[i], 1);
    }
    ctl->abort = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(&ctl->tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  pdl_wait();                       // the previous launch's results are visible from here on

  ProducerLog plog;
  if (warp < 4) {
    softmax_role<T, Cfg, DV>(p, ctl, tmem);
  } else if (warp == 4) {
    if ((threadIdx.x & 31) == 0) producer_role<Cfg>(p, smem, ctl, plog);
  } else {
    if ((threadIdx.x & 31) == 0) mma_role<Cfg>(p, smem, ctl, tmem);
  }
  pdl_trigger();

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  } else if (warp == 4 && (threadIdx.x & 31) == 0) {
    producer_drain(p, ctl, plog, Cfg::kStages, Cfg::kStages);
  }
}

template <typename T, int DQK, int DROPE, int DV>
cudaError_t launch_attn(const AttnParams &p, int grid, cudaStream_t stream) {
  using Cfg = AttnCfg<T, DQK, DROPE, DV>;
  auto kern = attn_fwd_kernel<T, DQK, DROPE, DV>;
  static SmemLimitRecord limit;       // this kernel's
  cudaError_t e = limit.ensure(kern, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), Cfg::kSmemBytes, stream, p);
}

}  // namespace wf
