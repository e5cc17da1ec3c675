// dca.cu -- dual chunk attention over the library's own kernels.
//
// "Dual Chunk Attention" (wiki article) splits a long sequence into chunks
// and attends within a chunk, to the neighbouring chunk and across chunks,
// each with its own remapping of relative positions; the article gives no
// formulas.  The reading taken here: the caller supplies each query in three
// forms, already rotated for the three position maps, and query i of chunk c
// scores key j <= i with q_intra (j in chunk c), q_succ (chunk c - 1) or
// q_inter (earlier chunks); one softmax over all of them.  That softmax is the
// merge (by log-sum-exp) of three attentions over disjoint key sets:
//   intra  -- packed sequences = the chunks, causal;
//   succ   -- packed, query chunk c against key chunk c - 1, no mask;
//   inter  -- per query chunk c >= 2, dense against keys [0, (c - 1) C);
// each writes its rows and LSE into a scratch part, and the merge pass
// combines the three parts into out (rows without a part keep LSE -inf).
#include <cmath>
#include <vector>

#include "attn_params.h"
#include "runtime.h"

using namespace wf;

namespace {

wf_tensor_t view(void *data, int32_t dtype, std::initializer_list<int64_t> shape,
                 std::initializer_list<int64_t> stride) {
  wf_tensor_t t{};
  t.data = data;
  t.dtype = dtype;
  t.ndim = static_cast<int32_t>(shape.size());
  int i = 0;
  for (int64_t x : shape) t.shape[i++] = x;
  i = 0;
  for (int64_t x : stride) t.stride[i++] = x;
  return t;
}

char *at(const wf_tensor_t *t, int64_t elems) {
  return static_cast<char *>(t->data) + elems * static_cast<int64_t>(dtype_size(t->dtype));
}

}  // namespace

extern "C" wf_status_t wf_attn_dca(const wf_tensor_t *qIntra, const wf_tensor_t *qSucc,
                                   const wf_tensor_t *qInter, const wf_tensor_t *k, const wf_tensor_t *v,
                                   int64_t chunkSize, int32_t headNum, int32_t kvHeadNum, float qkScale,
                                   wf_tensor_t *out, wf_tensor_t *lse, void *stream) {
  clear_error();
  wf_status_t st;
  if (!qIntra || !qSucc || !qInter || !k || !v || !out)
    return fail(WF_ERR_INVALID_ARG, "qIntra, qSucc, qInter, k, v and out are required");
  const int32_t dt = qIntra->dtype;
  if (dt != WF_BF16 && dt != WF_F16)
    return fail(WF_ERR_UNSUPPORTED, "dual chunk attention takes WF_BF16 or WF_F16 inputs");
  if (chunkSize <= 0) return fail(WF_ERR_INVALID_ARG, "chunkSize must be positive");
  for (const wf_tensor_t *t : {qIntra, qSucc, qInter, k, v, static_cast<const wf_tensor_t *>(out)})
    if ((st = check_tensor(t, "dca tensor", 4, dt, true)) != WF_OK) return st;
  const int64_t B = qIntra->shape[0], H = qIntra->shape[1], L = qIntra->shape[2], D = qIntra->shape[3];
  const int64_t Dv = v->shape[3];
  for (const wf_tensor_t *t : {qSucc, qInter})
    for (int i = 0; i < 4; ++i)
      if (t->shape[i] != qIntra->shape[i]) return fail(WF_ERR_INVALID_ARG, "the three query forms differ in shape");
  if (H != headNum || k->shape[1] != kvHeadNum || v->shape[1] != kvHeadNum || k->shape[0] != B ||
      v->shape[0] != B || k->shape[2] != L || v->shape[2] != L || k->shape[3] != D)
    return fail(WF_ERR_INVALID_ARG, "k / v must be [B, kvHeadNum, L, D] beside q [B, headNum, L, D]");
  if (out->shape[0] != B || out->shape[1] != H || out->shape[2] != L || out->shape[3] != Dv)
    return fail(WF_ERR_INVALID_ARG, "out must be [B, headNum, L, Dv]");
  if (lse) {
    if ((st = check_tensor(lse, "lse", 3, WF_F32, false)) != WF_OK) return st;
    if (lse->shape[0] != B || lse->shape[1] != H || lse->shape[2] != L)
      return fail(WF_ERR_INVALID_ARG, "lse must be [B, headNum, L]");
  }
  if (B == 0 || L == 0) return WF_OK;
  if (Dv % 8 != 0) return fail(WF_ERR_UNSUPPORTED, "Dv must be a multiple of 8");
  if (!current_device_state(&st)) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  // Scratch: 3 parts [L][H][Dv] (input type), their LSE [3][L][H] fp32, lengths.
  const int64_t nc = (L + chunkSize - 1) / chunkSize;
  const int64_t rows = L * H;
  const size_t es = dtype_size(dt);
  const size_t part_bytes = ((size_t)(3 * rows * Dv) * es + 255) & ~size_t(255);
  const size_t lse_bytes = ((size_t)(3 * rows) * 4 + 255) & ~size_t(255);
  const size_t len_bytes = (size_t)(3 * nc) * 4;
  void *scr = nullptr;
  if ((st = stream_scratch(cs, part_bytes + lse_bytes + len_bytes, &scr)) != WF_OK) return st;
  char *parts = static_cast<char *>(scr);
  float *lses = reinterpret_cast<float *>(parts + part_bytes);
  int32_t *lens = reinterpret_cast<int32_t *>(parts + part_bytes + lse_bytes);
  // lens: [0, nc) chunk lengths, [nc, 2nc - 1) lengths of chunks 1.., [2nc, 3nc - 1) C
  std::vector<int32_t> h_len(3 * nc, static_cast<int32_t>(chunkSize));
  for (int64_t c = 0; c < nc; ++c) h_len[c] = static_cast<int32_t>(std::min(chunkSize, L - c * chunkSize));
  for (int64_t c = 1; c < nc; ++c) h_len[nc + c - 1] = h_len[c];
  cudaError_t e = cudaMemcpyAsync(lens, h_len.data(), len_bytes, cudaMemcpyHostToDevice, cs);
  if (e != cudaSuccess) return cuda_fail(e, "copying the chunk lengths");

  for (int64_t b = 0; b < B; ++b) {
    // parts 1 and 2 start without a contribution (LSE -inf) on every row
    if ((e = launch_fill_f32(lses + rows, 2 * rows, -INFINITY, cs)) != cudaSuccess)
      return cuda_fail(e, "filling the LSE parts");
    const int64_t q_off = b * qIntra->stride[0], k_off = b * k->stride[0], v_off = b * v->stride[0];
    auto q_tok = [&](const wf_tensor_t *q, int64_t t0, int64_t n) {     // [n, H, D] from token t0
      return view(at(q, b * q->stride[0] + t0 * q->stride[2]), dt, {n, H, D}, {q->stride[2], q->stride[1], 1});
    };
    auto kv_tok = [&](const wf_tensor_t *t, int64_t t0, int64_t n, int64_t d, int64_t off) {
      return view(at(t, off + t0 * t->stride[2]), dt, {n, kvHeadNum, d}, {t->stride[2], t->stride[1], 1});
    };
    auto part_tok = [&](int p, int64_t t0, int64_t n) {                 // [n, H, Dv] of part p
      return view(parts + ((size_t)p * rows + t0 * H) * Dv * es, dt, {n, H, Dv}, {H * Dv, Dv, 1});
    };
    auto lse_tok = [&](int p, int64_t t0, int64_t n) {
      return view(lses + p * rows + t0 * H, WF_F32, {n, H}, {H, 1});
    };
    // intra: every chunk against itself, causal
    {
      wf_tensor_t q = q_tok(qIntra, 0, L), kk = kv_tok(k, 0, L, D, k_off), vv = kv_tok(v, 0, L, Dv, v_off);
      wf_tensor_t ql = view(lens, WF_I32, {nc}, {1});
      wf_tensor_t o = part_tok(0, 0, L), l = lse_tok(0, 0, L);
      if ((st = wf_attn_fwd_ex(&q, nullptr, &kk, nullptr, &vv, &ql, &ql, nullptr, headNum, kvHeadNum,
                               qkScale, WF_MASK_CAUSAL, &o, &l, 1, stream)) != WF_OK)
        return st;
    }
    // succ: chunk c >= 1 against chunk c - 1, all of it visible
    if (nc >= 2) {
      const int64_t nq = L - chunkSize, nk = (nc - 1) * chunkSize;
      wf_tensor_t q = q_tok(qSucc, chunkSize, nq), kk = kv_tok(k, 0, nk, D, k_off),
                  vv = kv_tok(v, 0, nk, Dv, v_off);
      wf_tensor_t ql = view(lens + nc, WF_I32, {nc - 1}, {1}), kl = view(lens + 2 * nc, WF_I32, {nc - 1}, {1});
      wf_tensor_t o = part_tok(1, chunkSize, nq), l = lse_tok(1, chunkSize, nq);
      if ((st = wf_attn_fwd_ex(&q, nullptr, &kk, nullptr, &vv, &ql, &kl, nullptr, headNum, kvHeadNum,
                               qkScale, WF_MASK_NONE, &o, &l, 1, stream)) != WF_OK)
        return st;
    }
    // inter: chunk c >= 2 against keys [0, (c - 1) C), one dense call each
    for (int64_t c = 2; c < nc; ++c) {
      const int64_t t0 = c * chunkSize, n = h_len[c], nk = (c - 1) * chunkSize;
      wf_tensor_t q = view(at(qInter, q_off + t0 * qInter->stride[2]), dt, {1, H, n, D},
                           {qInter->stride[0], qInter->stride[1], qInter->stride[2], 1});
      wf_tensor_t kk = view(at(k, k_off), dt, {1, kvHeadNum, nk, D}, {k->stride[0], k->stride[1], k->stride[2], 1});
      wf_tensor_t vv = view(at(v, v_off), dt, {1, kvHeadNum, nk, Dv}, {v->stride[0], v->stride[1], v->stride[2], 1});
      wf_tensor_t o = view(parts + ((size_t)2 * rows + t0 * H) * Dv * es, dt, {1, H, n, Dv},
                           {rows * Dv, Dv, H * Dv, 1});
      wf_tensor_t l = view(lses + 2 * rows + t0 * H, WF_F32, {1, H, n}, {rows, 1, H});
      if ((st = wf_attn_fwd_ex(&q, nullptr, &kk, nullptr, &vv, nullptr, nullptr, nullptr, headNum, kvHeadNum,
                               qkScale, WF_MASK_NONE, &o, &l, 0, stream)) != WF_OK)
        return st;
    }
    // merge the three parts of every row (row r = token * H + head) into out[b]
    MergeParams mp{};
    mp.parts = parts;
    mp.parts_type = elem_type_of(dt);
    mp.p_ss = rows * Dv;
    mp.p_sr = Dv;
    mp.lses = lses;
    mp.l_ss = rows;
    mp.l_sr = 1;
    mp.n_split = 3;
    mp.dv = static_cast<int32_t>(Dv);
    mp.rows = rows;
    mp.n1 = L;
    mp.n2 = H;
    mp.out = at(out, b * out->stride[0]);
    mp.out_type = elem_type_of(dt);
    mp.o_s1 = out->stride[2];
    mp.o_s2 = out->stride[1];
    if (lse) {
      mp.lse = reinterpret_cast<float *>(at(lse, b * lse->stride[0]));
      mp.e_s1 = lse->stride[2];
      mp.e_s2 = lse->stride[1];
    }
    if ((e = launch_merge(mp, cs)) != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return WF_OK;
}
