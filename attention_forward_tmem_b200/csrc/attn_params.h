// attn_params.h -- kernel parameter block and launch table shared by the
// attention kernels and the host runtime (internal; not part of the C ABI).
#pragma once
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace wf {

constexpr int kBlockM = 128;     // query rows per tile (one TMEM lane per row)
constexpr int kBlockN = 128;     // keys per KV tile
constexpr int kThreads = 192;    // warps 0-3 softmax, warp 4 TMA, warp 5 MMA

enum MaskKind : int32_t { kMaskNone = 0, kMaskCausal = 1, kMaskKeep = 2, kMaskAdd = 3 };
enum MaskDtype : int32_t { kMaskU8 = 0, kMaskF32 = 1, kMaskBF16 = 2, kMaskF16 = 3 };
// Element types of the kernels and the merge pass.
enum ElemType : int32_t { kElemF32 = 0, kElemBF16 = 1, kElemF16 = 2 };

// Device status codes (same numbers as wf_status_t).
constexpr int32_t kDevInvalidArg = 1;
constexpr int32_t kDevTimeout = 6;

// Debug switches for the bounded-wait test entry point (0 in production).
constexpr uint32_t kDebugStarveFirstK = 1u;   // producer never loads the first K tile

// Work order.  A work item is (sequence b, query head h, unit u), a unit being
// `unit_rows` consecutive query rows.  Items are enumerated sequence by
// sequence (packed: longest sequence first), then by kv head, then by unit
// (causal: the longest unit first), with the query heads of one GQA group
// adjacent: the items running at the same time on the 148 SMs then share
// few K/V tensors, which stay in L2, and the short units come last.
//
// Packed-sequence schedule workspace (int32 words), written by sched_prep:
//   [0] number of work items, [1] length-check flag,
//   [cu_q .. cu_q+B] and [cu_k .. cu_k+B] prefix sums of the lengths,
//   [order .. order+B) sequences by unit count, longest first,
//   [cu_work .. cu_work+B] prefix sums of (units x headNum) in that order.
struct SchedLayout {
  int32_t cu_q, cu_k, order, cu_work;   // offsets in words
  int64_t words;
};

struct alignas(64) AttnParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_qr, tm_kr;   // 4-d maps (D, rows, heads, batch);
                                                 // fp32: tm_v maps V^T (rows, D, heads, batch)
  // Fused cache write (two-tile kernel, dense, no mask): key rows
  // [fuse_lo, fuse_hi) of K / V are read from tm_kc / tm_vc (the new chunk,
  // row - fuse_lo) instead of tm_k / tm_v, and the CTAs of the first unit of
  // each kv head store them into tm_k / tm_v.  fuse_hi == 0: no fusion.
  CUtensorMap tm_kc, tm_vc;
  int32_t fuse_lo, fuse_hi;
  // Dense output through TMA stores (tma_out != 0): map of out (Dv, Lq, Hq,
  // B) with 64 x 32 boxes; the kernel uses it where it has the staging area.
  CUtensorMap tm_o;
  int32_t tma_out;
  // Split-KV partial rows through TMA stores (tma_part != 0, dense): map of
  // part_o (Dv, part_rows, n_split) in fp32 with 32 x 32 boxes.
  CUtensorMap tm_po;
  int32_t tma_part;
  void *out;
  int64_t o_sb, o_sh, o_si;                      // element strides of out (batch, head, row)
  const void *mask;
  int64_t m_sb, m_sh, m_si, m_sj;                // element strides of the mask (0 = broadcast)
  int32_t mask_kind, mask_dtype;
  int32_t causal_top_left;                      // causal: key j visible to row i iff j <= i
  int32_t batch, hq, hkv, group;
  int32_t lq, lk;                                // dense lengths
  int32_t varlen;
  int32_t kv_padded;                             // packed q, K/V [batch, max_seq, heads, D]
  int32_t unit_rows;                             // query rows per work unit (128 or 256)
  int32_t n_units_dense, units_per_bh;           // dense: total units, units per (b, h)
  int32_t unit_major;                            // dense: the last unit_major (batch, kv head)
                                                 // blocks claimed by unit rank (unit_major_item)
  const int32_t *ws;                             // varlen schedule (device)
  int32_t *counters;                             // two-tile kernel: [next item, CTAs done],
                                                 // zero before a launch, zero after it
  SchedLayout sl;
  // Split-KV: with n_split > 1 every unit's KV tiles are dealt into n_split
  // contiguous ranges, one work item each (item = unit * n_split + split);
  // each writes its rows normalised over its own keys, in fp32, to
  // part_o [n_split][part_rows][DV] and their natural-log LSE to
  // part_lse [n_split][part_rows], and a merge pass combines them.  Row index:
  // dense ((b * hq + h) * lq + i), packed (token * hq + h).
  int32_t n_split;
  float *part_o, *part_lse;
  int64_t part_rows;
  // Optional natural-log LSE of every row (n_split <= 1 only; NULL = none),
  // element strides (batch, head, row) as for out.
  float *lse;
  int64_t l_sb, l_sh, l_si;
  float scale_log2;                              // qkScale * log2(e)
  int32_t *status;                               // device status word
  long long timeout_cycles;
  uint32_t debug_flags;
};

using AttnLaunchFn = cudaError_t (*)(const AttnParams &, int grid, cudaStream_t);

// Generation of the per-device settings (raised by wf_shutdown, after which a
// device may have been reset): a kernel's shared-memory limit is set once per
// device and generation instead of before every launch.
extern std::atomic<uint32_t> g_setup_generation;

// One record per kernel (a static of each kernel's launch function).
struct SmemLimitRecord {
  std::atomic<uint32_t> done[64];     // generation in which each device was set
  template <typename K>
  cudaError_t ensure(K kern, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint32_t gen = g_setup_generation.load(std::memory_order_acquire);
    std::atomic<uint32_t> *slot = dev >= 0 && dev < 64 ? &done[dev] : nullptr;
    if (slot && slot->load(std::memory_order_acquire) == gen) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && slot) slot->store(gen, std::memory_order_release);
    return e;
  }
};

// Launch with programmatic stream serialization: the kernel may begin (its
// prologue) while the previous launch on the stream finishes; every kernel of
// the library waits (pdl_wait) before it touches global memory, and signals
// (pdl_trigger) once its own work is done.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

struct AttnKernel {
  AttnLaunchFn launch;
  int32_t unit_rows;     // query rows per work unit of this kernel
};

// Instances of the 16-bit kernel: no mask or the in-kernel causal mask; the
// same plus the write of a BlockKVCache chunk; explicit masks (boolean keep
// or additive) read from memory.  Each instance carries only its own code:
// with the explicit-mask paths compiled into the causal instance, ~20% of its
// executed instructions were predicated-off mask address arithmetic.
enum KernelKind : int32_t { kKindPlain = 0, kKindFuse = 1, kKindMask = 2 };

// Kernel for (ElemType, dqk, drope, dv, kind); launch == nullptr if none.
AttnKernel find_attn_kernel(int dtype, int dqk, int drope, int dv, int kind = kKindPlain);

// V [rows, heads, batch] x d (element strides) -> V^T [batch][heads][d][ld] (fp32).
cudaError_t launch_transpose_v(const float *v, int64_t s_row, int64_t s_head, int64_t s_batch,
                               int32_t rows, int32_t heads, int32_t batch, int32_t d, float *vt,
                               int64_t ld, cudaStream_t stream);

// Merge of per-key-set partial results by their LSE (merge.cu).  Row r of
// the output decomposes as r = (i0 * n1 + i1) * n2 + i2.
struct MergeParams {
  const void *parts;         // [n_split][rows][dv], element strides ss / sr
  int32_t parts_type;        // ElemType
  int64_t p_ss, p_sr;
  const float *lses;         // [n_split][rows], element strides
  int64_t l_ss, l_sr;
  int32_t n_split, dv;
  int64_t rows, n1, n2;
  const int32_t *sched;      // packed schedule words (or NULL): nothing is merged if
  int32_t sched_tokens;      // the length check failed (word 1), and only rows below
                             // sched[sched_tokens] * n2 (the sequences' tokens) are
  void *out;
  int32_t out_type;          // ElemType
  int64_t o_s0, o_s1, o_s2;
  float *lse;                // NULL: not wanted
  int64_t e_s0, e_s1, e_s2;
};

cudaError_t launch_merge(const MergeParams &mp, cudaStream_t stream);

// k_max_len: padded K/V, the longest kv length that fits (else any value
// >= n_k_tokens); lengths above it are rejected like sums past the tensors.
cudaError_t launch_sched_prep(const int32_t *q_len, const int32_t *k_len, int32_t batch,
                              int64_t n_q_tokens, int64_t n_k_tokens, int64_t k_max_len,
                              int32_t head_num,
                              int32_t unit_rows, int32_t *ws, const SchedLayout &sl,
                              int32_t *status, cudaStream_t stream);

}  // namespace wf
