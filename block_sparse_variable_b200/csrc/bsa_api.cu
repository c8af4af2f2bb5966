// bsa_api.cu -- host side of the C ABI declared in include/bsa.h:
// descriptor validation (the first phase of the two-phase interface),
// workspace sizing and carving, and the launch sequence of each pass.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "bsa_internal.h"

namespace bsa {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace bsa

namespace {

using bsa::Problem;

struct Args {
  const bsa_tensor *q, *k, *v, *index, *cu_q, *cu_kv, *seqused, *bt, *out, *lse;
  const bsa_tensor *dout, *dq, *dk, *dv;
  const bsa_params *prm;
  bool bwd;
};

bool present(const bsa_tensor *t) { return t != nullptr && t->data != nullptr; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool block_ok(int64_t x) { return x == 128 || x == 256 || x == 512 || x == 1024; }

// A dense-value tensor (q/k/v/out/...): given ndim, dtype, last stride 1, the
// other strides 16-byte multiples (8 16-bit or 16 8-bit elements) and a
// 16-byte-aligned base (16-byte vector loads and TMA boxes start on 16-byte
// boundaries).
bsa_status check_values(const bsa_tensor *t, int ndim, int dtype) {
  if (t->ndim != ndim || t->dtype != dtype) return BSA_ERR_PARAM_INVALID;
  if (t->stride[ndim - 1] != 1) return BSA_ERR_PARAM_INVALID;
  const int64_t per16 = dtype == BSA_F8E4M3 ? 16 : 8;
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return BSA_ERR_PARAM_INVALID;
    if (i < ndim - 1 && (t->stride[i] % per16 != 0 || t->stride[i] < 0)) return BSA_ERR_PARAM_INVALID;
  }
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0) return BSA_ERR_PARAM_INVALID;
  return BSA_OK;
}

bool same_shape(const bsa_tensor *a, const bsa_tensor *b) {
  if (a->ndim != b->ndim || a->dtype != b->dtype) return false;
  for (int i = 0; i < a->ndim; ++i)
    if (a->shape[i] != b->shape[i]) return false;
  return true;
}

bool vec_ok(const bsa_tensor *t, int dtype, int64_t n) {
  return t->ndim == 1 && t->dtype == dtype && t->shape[0] == n && (n <= 1 || t->stride[0] == 1);
}

struct Layout {
  bsa_ws_layout pub;
  // private regions
  bsa_ws_region row_batch, kb_batch, sorted, inv_cnt, inv_sub;
};

uint64_t place(uint64_t &cur, uint64_t bytes, bsa_ws_region &r) {
  cur = (cur + 255) & ~uint64_t(255);
  r.offset = cur;
  r.bytes = bytes;
  cur += bytes;
  return r.offset;
}

// Validates every descriptor and fills the problem sizes, tensor views and
// workspace layout.  Returns BSA_OK with p.B == 0 ... for an empty problem.
bsa_status prepare(const Args &a, Problem &p, Layout &L, bool &empty) {
  std::memset(&p, 0, sizeof(p));
  std::memset(&L, 0, sizeof(L));
  empty = false;
  if (!a.prm || !a.q || !a.k || !a.v || !a.index || !a.out) return BSA_ERR_NULLPTR;
  if (!a.q->data || !a.k->data || !a.v->data || !a.index->data || !a.out->data)
    return BSA_ERR_NULLPTR;
  if (a.bwd && (!present(a.dout) || !present(a.lse) || !present(a.dq) || !present(a.dk) ||
                !present(a.dv)))
    return BSA_ERR_NULLPTR;
  const bsa_params &P = *a.prm;
  const int ql = P.q_layout, kl = P.kv_layout;
  if (!((ql == BSA_LAYOUT_BNSD && kl == BSA_LAYOUT_BNSD) ||
        (ql == BSA_LAYOUT_TND && (kl == BSA_LAYOUT_TND || kl == BSA_LAYOUT_PA_BBND))))
    return BSA_ERR_PARAM_INVALID;
  const int dt = a.q->dtype;
  if (dt != BSA_F16 && dt != BSA_BF16 && dt != BSA_F8E4M3) return BSA_ERR_PARAM_INVALID;
  const bool fp8 = dt == BSA_F8E4M3;
  if (fp8 && a.bwd) return BSA_ERR_UNSUPPORTED;  // the backward takes 16-bit inputs
  // FP8 inputs write a 16-bit out whose dtype is the caller's choice
  const int odt = fp8 ? a.out->dtype : dt;
  if (odt != BSA_F16 && odt != BSA_BF16) return BSA_ERR_PARAM_INVALID;
  const int qnd = ql == BSA_LAYOUT_BNSD ? 4 : 3;
  const int knd = kl == BSA_LAYOUT_TND ? 3 : 4;
  bsa_status st;
  if ((st = check_values(a.q, qnd, dt)) != BSA_OK) return st;
  if ((st = check_values(a.k, knd, dt)) != BSA_OK) return st;
  if ((st = check_values(a.v, knd, dt)) != BSA_OK) return st;
  if ((st = check_values(a.out, qnd, odt)) != BSA_OK) return st;
  if (a.out->ndim != a.q->ndim || !same_shape(a.k, a.v)) return BSA_ERR_PARAM_INVALID;
  for (int i = 0; i < a.q->ndim; ++i)
    if (a.out->shape[i] != a.q->shape[i]) return BSA_ERR_PARAM_INVALID;
  if (a.bwd) {
    if ((st = check_values(a.dout, qnd, dt)) != BSA_OK) return st;
    if ((st = check_values(a.dq, qnd, dt)) != BSA_OK) return st;
    if ((st = check_values(a.dk, knd, dt)) != BSA_OK) return st;
    if ((st = check_values(a.dv, knd, dt)) != BSA_OK) return st;
    if (!same_shape(a.q, a.dout) || !same_shape(a.q, a.dq) || !same_shape(a.k, a.dk) ||
        !same_shape(a.k, a.dv))
      return BSA_ERR_PARAM_INVALID;
  }

  const int64_t N1 = ql == BSA_LAYOUT_BNSD ? a.q->shape[1] : a.q->shape[1];
  const int64_t D = a.q->shape[qnd - 1];
  const int64_t N2 = P.num_kv_heads == 0 ? P.num_heads : P.num_kv_heads;
  if (P.num_heads != N1 || N2 <= 0 || N1 % N2 != 0) return BSA_ERR_PARAM_INVALID;
  if (a.k->shape[knd - 1] != D) return BSA_ERR_PARAM_INVALID;
  if (D != 64 && D != 128) return BSA_ERR_UNSUPPORTED;
  if (fp8 && D != 128) return BSA_ERR_UNSUPPORTED;  // one 128-byte box per row
  const int64_t BQ = P.block_shape[0], BKV = P.block_shape[1];
  if (!block_ok(BQ) || !block_ok(BKV)) return BSA_ERR_PARAM_INVALID;
  if (!(P.scale >= 0.0) || std::isinf(P.scale)) return BSA_ERR_PARAM_INVALID;

  int64_t B = 0, Sq = 0, Skv = 0, Tq = 0, Tkv = 0, page = 0, max_pages = 0, num_pages = 0;
  if (ql == BSA_LAYOUT_BNSD) {
    B = a.q->shape[0];
    Sq = a.q->shape[2];
    Skv = a.k->shape[2];
    if (a.k->shape[0] != B || a.k->shape[1] != N2) return BSA_ERR_PARAM_INVALID;
    if (present(a.cu_q) || present(a.cu_kv) || present(a.bt)) return BSA_ERR_PARAM_INVALID;
  } else {
    if (!present(a.cu_q)) return BSA_ERR_NULLPTR;
    if (a.cu_q->ndim != 1 || a.cu_q->shape[0] < 1) return BSA_ERR_PARAM_INVALID;
    B = a.cu_q->shape[0] - 1;
    if (!vec_ok(a.cu_q, BSA_I64, B + 1)) return BSA_ERR_PARAM_INVALID;
    Tq = a.q->shape[0];
    if (kl == BSA_LAYOUT_TND) {
      if (!present(a.cu_kv)) return BSA_ERR_NULLPTR;
      if (!vec_ok(a.cu_kv, BSA_I64, B + 1)) return BSA_ERR_PARAM_INVALID;
      if (present(a.bt)) return BSA_ERR_PARAM_INVALID;
      Tkv = a.k->shape[0];
      if (a.k->shape[1] != N2) return BSA_ERR_PARAM_INVALID;
    } else {
      if (present(a.cu_kv)) return BSA_ERR_PARAM_INVALID;
      if (!present(a.bt) || !present(a.seqused)) return BSA_ERR_NULLPTR;
      num_pages = a.k->shape[0];
      page = a.k->shape[1];
      if (a.k->shape[2] != N2) return BSA_ERR_PARAM_INVALID;
      if (page <= 0 || page % 128 != 0) return BSA_ERR_UNSUPPORTED;
      if (a.bt->ndim != 2 || a.bt->dtype != BSA_I32 || a.bt->shape[0] != B ||
          a.bt->shape[1] < 1 || (a.bt->shape[1] > 1 && a.bt->stride[1] != 1))
        return BSA_ERR_PARAM_INVALID;
      max_pages = a.bt->shape[1];
    }
  }
  if (present(a.seqused) && !vec_ok(a.seqused, BSA_I32, B)) return BSA_ERR_PARAM_INVALID;

  // index
  const bsa_tensor *ix = a.index;
  int64_t Hidx = 0, R = 0, W = 0;
  if (ix->dtype != BSA_U16) return BSA_ERR_PARAM_INVALID;
  if (ql == BSA_LAYOUT_BNSD) {
    if (ix->ndim != 4 || ix->shape[0] != B || ix->shape[2] != cdiv(Sq, BQ))
      return BSA_ERR_PARAM_INVALID;
    Hidx = ix->shape[1];
    R = ix->shape[2];
    W = ix->shape[3];
  } else {
    if (ix->ndim != 3) return BSA_ERR_PARAM_INVALID;
    Hidx = ix->shape[0];
    R = ix->shape[1];
    W = ix->shape[2];
  }
  if (Hidx != N1 && Hidx != N2) return BSA_ERR_PARAM_INVALID;
  if (W < 1 || W > 65535 || R < 0 || ix->stride[ix->ndim - 1] != 1) return BSA_ERR_PARAM_INVALID;

  // lse
  if (P.mask_type != BSA_MASK_NONE && P.mask_type != BSA_MASK_CAUSAL) return BSA_ERR_PARAM_INVALID;
  const bool want_lse = a.bwd || P.return_lse;
  if (want_lse) {
    if (!present(a.lse)) return BSA_ERR_NULLPTR;
    const bsa_tensor *l = a.lse;
    if (l->dtype != BSA_F32) return BSA_ERR_PARAM_INVALID;
    if (ql == BSA_LAYOUT_BNSD) {
      if (l->ndim != 3 || l->shape[0] != B || l->shape[1] != N1 || l->shape[2] != Sq)
        return BSA_ERR_PARAM_INVALID;
    } else {
      if (l->ndim != 2 || l->shape[0] != Tq || l->shape[1] != N1) return BSA_ERR_PARAM_INVALID;
    }
    if (reinterpret_cast<uintptr_t>(l->data) % 4 != 0) return BSA_ERR_PARAM_INVALID;
  }

  // ---- sizes
  const int64_t rows_q = ql == BSA_LAYOUT_BNSD ? B * Sq : Tq;
  if (B == 0 || rows_q == 0 || N1 == 0) {
    empty = true;
    return BSA_OK;
  }
  const int64_t Rg = ql == BSA_LAYOUT_BNSD ? B * R : R;
  int64_t tk_max;
  if (kl == BSA_LAYOUT_BNSD) tk_max = B * cdiv(Skv, BKV);
  else if (kl == BSA_LAYOUT_TND) tk_max = cdiv(Tkv, BKV) + B;
  else tk_max = B * cdiv(max_pages * page, BKV);
  const int64_t nsub = BQ / 128, ksl = BKV / 128;
  const int64_t fwd_slots = N1 * Rg * nsub;
  const int64_t bwd_slots = N2 * tk_max * ksl;
  const int64_t lim = int64_t(1) << 30;
  if (fwd_slots >= lim || bwd_slots >= lim || Hidx * Rg * W >= (int64_t(1) << 34) ||
      Hidx * tk_max >= lim || B >= lim)
    return BSA_ERR_UNSUPPORTED;
  const int64_t fpad = cdiv(fwd_slots, bsa::kSortChunk) * bsa::kSortChunk;
  const int64_t bpad = cdiv(bwd_slots, bsa::kSortChunk) * bsa::kSortChunk;

  // ---- fill the problem
  p.B = int32_t(B); p.N1 = int32_t(N1); p.N2 = int32_t(N2); p.D = int32_t(D);
  p.g = int32_t(N1 / N2); p.Hidx = int32_t(Hidx); p.BQ = int32_t(BQ); p.BKV = int32_t(BKV);
  p.W = int32_t(W); p.nsub = int32_t(nsub); p.ksl = int32_t(ksl);
  p.q_layout = ql; p.kv_layout = kl; p.dtype = dt; p.out_dtype = odt;
  p.Sq = Sq; p.Skv = Skv; p.Tq = Tq; p.Tkv = Tkv;
  p.R = int32_t(R); p.Rg = int32_t(Rg); p.tk_max = int32_t(tk_max);
  p.page_size = int32_t(page); p.max_pages = int32_t(max_pages); p.num_pages = int32_t(num_pages);
  p.rows_q = rows_q;
  const double scale = P.scale == 0.0 ? 1.0 / std::sqrt(double(D)) : P.scale;
  p.scale = float(scale);
  p.scale_log2 = float(scale * 1.4426950408889634);
  p.return_lse = want_lse ? 1 : 0;
  p.causal = P.mask_type == BSA_MASK_CAUSAL ? 1 : 0;
  p.deterministic = a.bwd && P.deterministic ? 1 : 0;
  // GenericBlockSparseAttention, attribute table, isPackedGQA: the q heads of
  // a group share the sparse pattern.  The forward then packs them into one
  // tile whenever 128 / g rows per head is a whole number of 8-row swizzle
  // atoms; the backward (kv-major) already streams K/V once per group.
  const int64_t g = N1 / N2;
  p.pack_g = (!a.bwd && Hidx == N2 && (g == 2 || g == 4 || g == 8 || g == 16)) ? int32_t(g) : 1;
  p.fsub = int32_t(nsub * p.pack_g);
  p.fwd_slots = fwd_slots; p.bwd_slots = bwd_slots;
  p.fwd_slots_pad = fpad; p.bwd_slots_pad = bpad;

  auto qview = [&](const bsa_tensor *t, int64_t &sb, int64_t &sh, int64_t &st) {
    if (ql == BSA_LAYOUT_BNSD) { sb = t->stride[0]; sh = t->stride[1]; st = t->stride[2]; }
    else { sb = 0; st = t->stride[0]; sh = t->stride[1]; }
  };
  auto kview = [&](const bsa_tensor *t, int64_t &sb, int64_t &sh, int64_t &st) {
    if (kl == BSA_LAYOUT_BNSD) { sb = t->stride[0]; sh = t->stride[1]; st = t->stride[2]; }
    else if (kl == BSA_LAYOUT_TND) { sb = 0; st = t->stride[0]; sh = t->stride[1]; }
    else { sb = t->stride[0]; st = t->stride[1]; sh = t->stride[2]; }
  };
  p.q = a.q->data; qview(a.q, p.q_sb, p.q_sh, p.q_st);
  p.k = a.k->data; kview(a.k, p.k_sb, p.k_sh, p.k_st);
  p.v = a.v->data; kview(a.v, p.v_sb, p.v_sh, p.v_st);
  p.out = a.out->data; qview(a.out, p.o_sb, p.o_sh, p.o_st);
  if (want_lse) {
    p.lse = static_cast<float *>(a.lse->data);
    if (ql == BSA_LAYOUT_BNSD) { p.l_sb = a.lse->stride[0]; p.l_sh = a.lse->stride[1]; p.l_st = a.lse->stride[2]; }
    else { p.l_sb = 0; p.l_st = a.lse->stride[0]; p.l_sh = a.lse->stride[1]; }
  }
  if (a.bwd) {
    p.dout = a.dout->data; qview(a.dout, p.do_sb, p.do_sh, p.do_st);
    p.dq = a.dq->data; qview(a.dq, p.dq_sb, p.dq_sh, p.dq_st);
    p.dk = a.dk->data; kview(a.dk, p.dk_sb, p.dk_sh, p.dk_st);
    p.dv = a.dv->data; kview(a.dv, p.dv_sb, p.dv_sh, p.dv_st);
  }
  p.index = static_cast<const uint16_t *>(ix->data);
  p.ix_s0 = ix->stride[0]; p.ix_s1 = ix->stride[1]; p.ix_s2 = ix->stride[2];
  p.cu_q = present(a.cu_q) ? static_cast<const int64_t *>(a.cu_q->data) : nullptr;
  p.cu_kv = present(a.cu_kv) ? static_cast<const int64_t *>(a.cu_kv->data) : nullptr;
  p.seqused_kv = present(a.seqused) ? static_cast<const int32_t *>(a.seqused->data) : nullptr;
  p.block_table = present(a.bt) ? static_cast<const int32_t *>(a.bt->data) : nullptr;
  p.bt_s0 = present(a.bt) ? a.bt->stride[0] : 0;

  // ---- workspace layout
  uint64_t cur = 0;
  bsa_ws_layout &W_ = L.pub;
  place(cur, bsa::kStWords * 4, W_.status);
  place(cur, uint64_t(B) * sizeof(bsa::BatchInfo), W_.batch);
  place(cur, uint64_t(Rg) * 4, L.row_batch);
  place(cur, uint64_t(tk_max) * 4, L.kb_batch);
  place(cur, uint64_t(Hidx) * Rg * W * 2, W_.comp);
  place(cur, uint64_t(Hidx) * Rg * 4, W_.ncomp);
  // the deterministic backward sorts both work lists through the key buffers
  const int64_t kpad = !a.bwd ? fpad : p.deterministic ? (fpad > bpad ? fpad : bpad) : bpad;
  place(cur, uint64_t(kpad) * 8, W_.sort_keys);
  place(cur, uint64_t(kpad) * 8, L.sorted);
  if (!a.bwd || p.deterministic) place(cur, uint64_t(fwd_slots) * 4, W_.fwd_items);
  if (a.bwd) {
    const int64_t nnz_max = Hidx * Rg * (W < tk_max ? W : tk_max);
    place(cur, uint64_t(Hidx) * tk_max * 4, L.inv_cnt);
    place(cur, uint64_t(Hidx) * tk_max * 4, L.inv_sub);
    place(cur, (uint64_t(Hidx) * tk_max + 1) * 4, W_.inv_off);
    place(cur, uint64_t(nnz_max) * 4, W_.inv_list);
    place(cur, uint64_t(bwd_slots) * 4, W_.bwd_items);
    place(cur, uint64_t(rows_q) * N1 * 4, W_.dsum);
    if (!p.deterministic) place(cur, uint64_t(rows_q) * N1 * D * 4, W_.dq_acc);
  }
  W_.Rg = Rg;
  W_.tk_max = tk_max;
  W_.total_bytes = (cur + 255) & ~uint64_t(255);
  return BSA_OK;
}

template <typename T>
T *at(void *ws, const bsa_ws_region &r) {
  return r.bytes ? reinterpret_cast<T *>(static_cast<char *>(ws) + r.offset) : nullptr;
}

void carve(Problem &p, const Layout &L, void *ws) {
  p.status = at<uint32_t>(ws, L.pub.status);
  p.batch = at<bsa::BatchInfo>(ws, L.pub.batch);
  p.row_batch = at<int32_t>(ws, L.row_batch);
  p.kb_batch = at<int32_t>(ws, L.kb_batch);
  p.comp = at<uint16_t>(ws, L.pub.comp);
  p.ncomp = at<int32_t>(ws, L.pub.ncomp);
  p.keys = at<uint64_t>(ws, L.pub.sort_keys);
  p.sorted = at<uint64_t>(ws, L.sorted);
  p.fwd_items = at<int32_t>(ws, L.pub.fwd_items);
  p.inv_cnt = at<int32_t>(ws, L.inv_cnt);
  p.inv_sub = at<int32_t>(ws, L.inv_sub);
  p.inv_off = at<int32_t>(ws, L.pub.inv_off);
  p.inv_list = at<int32_t>(ws, L.pub.inv_list);
  p.bwd_items = at<int32_t>(ws, L.pub.bwd_items);
  p.dsum = at<float>(ws, L.pub.dsum);
  p.dq_acc = at<float>(ws, L.pub.dq_acc);
}

bsa_status check_ws(const Layout &L, void *ws, size_t bytes) {
  if (L.pub.total_bytes == 0) return BSA_OK;
  if (!ws || bytes < L.pub.total_bytes || reinterpret_cast<uintptr_t>(ws) % 256 != 0)
    return BSA_ERR_WORKSPACE;
  return BSA_OK;
}

#define BSA_LAUNCH(x)                          \
  do {                                         \
    if ((x) != cudaSuccess) return BSA_ERR_CUDA; \
  } while (0)

// events to record around the next call's main kernel (bsa_set_main_kernel_events)
thread_local cudaEvent_t t_ev_before = nullptr, t_ev_after = nullptr;

// takes the pending event pair of this host thread (at most one call uses it)
void take_events(cudaEvent_t &before, cudaEvent_t &after) {
  before = t_ev_before;
  after = t_ev_after;
  t_ev_before = t_ev_after = nullptr;
}

}  // namespace

namespace bsa {
void drop_pending_events() {
  cudaEvent_t a, b;
  take_events(a, b);
}
}  // namespace bsa

namespace {

bsa_status run_fwd(const Problem &p, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  BSA_LAUNCH(bsa::launch_prep_geometry(p, s));
  BSA_LAUNCH(bsa::launch_prep_compact(p, true, s));
  BSA_LAUNCH(bsa::launch_sort_items(p, p.fwd_slots_pad, p.fwd_items, s));
  if (e0) BSA_LAUNCH(cudaEventRecord(e0, s));
  BSA_LAUNCH(bsa::launch_fwd_main(p, s));
  if (e1) BSA_LAUNCH(cudaEventRecord(e1, s));
  return BSA_OK;
}

bsa_status run_bwd(const Problem &p, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  BSA_LAUNCH(bsa::launch_prep_geometry(p, s));
  // deterministic: the forward work list too (for the q-major dQ pass),
  // sorted before the backward keys reuse the key buffers
  BSA_LAUNCH(bsa::launch_prep_compact(p, p.deterministic != 0, s));
  if (p.deterministic) BSA_LAUNCH(bsa::launch_sort_items(p, p.fwd_slots_pad, p.fwd_items, s));
  BSA_LAUNCH(bsa::launch_prep_inverse(p, s));
  BSA_LAUNCH(bsa::launch_sort_items(p, p.bwd_slots_pad, p.bwd_items, s));
  BSA_LAUNCH(bsa::launch_bwd_pre(p, s));
  if (e0) BSA_LAUNCH(cudaEventRecord(e0, s));
  BSA_LAUNCH(bsa::launch_bwd_main(p, s));
  if (p.deterministic) BSA_LAUNCH(bsa::launch_dq_main(p, s));  // inside the events: both main kernels
  if (e1) BSA_LAUNCH(cudaEventRecord(e1, s));
  BSA_LAUNCH(bsa::launch_bwd_post(p, s));
  return BSA_OK;
}

Args fwd_args(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
              const bsa_tensor *index, const bsa_tensor *cu_q, const bsa_tensor *cu_kv,
              const bsa_tensor *seqused, const bsa_tensor *bt, const bsa_params *prm,
              const bsa_tensor *out, const bsa_tensor *lse) {
  Args a{};
  a.q = q; a.k = k; a.v = v; a.index = index; a.cu_q = cu_q; a.cu_kv = cu_kv;
  a.seqused = seqused; a.bt = bt; a.prm = prm; a.out = out; a.lse = lse; a.bwd = false;
  return a;
}

Args bwd_args(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
              const bsa_tensor *out, const bsa_tensor *dout, const bsa_tensor *lse,
              const bsa_tensor *index, const bsa_tensor *cu_q, const bsa_tensor *cu_kv,
              const bsa_tensor *seqused, const bsa_tensor *bt, const bsa_params *prm,
              const bsa_tensor *dq, const bsa_tensor *dk, const bsa_tensor *dv) {
  Args a = fwd_args(q, k, v, index, cu_q, cu_kv, seqused, bt, prm, out, lse);
  a.dout = dout; a.dq = dq; a.dk = dk; a.dv = dv; a.bwd = true;
  return a;
}

}  // namespace

extern "C" {

bsa_status bsa_set_main_kernel_events(void *before, void *after) {
  if ((before == nullptr) != (after == nullptr)) return BSA_ERR_NULLPTR;
  t_ev_before = static_cast<cudaEvent_t>(before);
  t_ev_after = static_cast<cudaEvent_t>(after);
  return BSA_OK;
}

int32_t bsa_abi_version(void) { return 3; }

const char *bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_NULLPTR: return "BSA_ERR_NULLPTR: a required pointer is NULL";
    case BSA_ERR_PARAM_INVALID: return "BSA_ERR_PARAM_INVALID: shapes, strides, dtypes or attributes disagree";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED: outside what this library supports";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE: workspace NULL, misaligned or too small";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA: a CUDA launch or call failed";
    case BSA_ERR_INNER: return "BSA_ERR_INNER: internal inconsistency";
  }
  return "unknown bsa_status";
}

bsa_status bsa_fwd_workspace_layout(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                    const bsa_tensor *index, const bsa_tensor *cu_q,
                                    const bsa_tensor *cu_kv, const bsa_tensor *seqused,
                                    const bsa_tensor *bt, const bsa_params *prm,
                                    const bsa_tensor *out, const bsa_tensor *lse,
                                    bsa_ws_layout *layout) {
  if (!layout) return BSA_ERR_NULLPTR;
  Problem p;
  Layout L;
  bool empty;
  bsa_status st = prepare(fwd_args(q, k, v, index, cu_q, cu_kv, seqused, bt, prm, out, lse), p, L, empty);
  if (st == BSA_OK) *layout = L.pub;
  return st;
}

bsa_status bsa_fwd_get_workspace(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                 const bsa_tensor *index, const bsa_tensor *cu_q,
                                 const bsa_tensor *cu_kv, const bsa_tensor *seqused,
                                 const bsa_tensor *bt, const bsa_params *prm,
                                 const bsa_tensor *out, const bsa_tensor *lse,
                                 size_t *workspace_bytes) {
  if (!workspace_bytes) return BSA_ERR_NULLPTR;
  bsa_ws_layout l;
  bsa_status st = bsa_fwd_workspace_layout(q, k, v, index, cu_q, cu_kv, seqused, bt, prm, out, lse, &l);
  if (st == BSA_OK) *workspace_bytes = size_t(l.total_bytes);
  return st;
}

bsa_status bsa_fwd(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                   const bsa_tensor *index, const bsa_tensor *cu_q, const bsa_tensor *cu_kv,
                   const bsa_tensor *seqused, const bsa_tensor *bt, const bsa_params *prm,
                   const bsa_tensor *out, const bsa_tensor *lse, void *workspace,
                   size_t workspace_bytes, void *stream) {
  cudaEvent_t e0, e1;
  take_events(e0, e1);
  Problem p;
  Layout L;
  bool empty;
  bsa_status st = prepare(fwd_args(q, k, v, index, cu_q, cu_kv, seqused, bt, prm, out, lse), p, L, empty);
  if (st != BSA_OK || empty) return st;
  if ((st = check_ws(L, workspace, workspace_bytes)) != BSA_OK) return st;
  carve(p, L, workspace);
  return run_fwd(p, static_cast<cudaStream_t>(stream), e0, e1);
}

bsa_status bsa_bwd_workspace_layout(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                    const bsa_tensor *out, const bsa_tensor *dout,
                                    const bsa_tensor *lse, const bsa_tensor *index,
                                    const bsa_tensor *cu_q, const bsa_tensor *cu_kv,
                                    const bsa_tensor *seqused, const bsa_tensor *bt,
                                    const bsa_params *prm, const bsa_tensor *dq,
                                    const bsa_tensor *dk, const bsa_tensor *dv,
                                    bsa_ws_layout *layout) {
  if (!layout) return BSA_ERR_NULLPTR;
  Problem p;
  Layout L;
  bool empty;
  bsa_status st = prepare(bwd_args(q, k, v, out, dout, lse, index, cu_q, cu_kv, seqused, bt, prm,
                                   dq, dk, dv), p, L, empty);
  if (st == BSA_OK) *layout = L.pub;
  return st;
}

bsa_status bsa_bwd_get_workspace(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                 const bsa_tensor *out, const bsa_tensor *dout,
                                 const bsa_tensor *lse, const bsa_tensor *index,
                                 const bsa_tensor *cu_q, const bsa_tensor *cu_kv,
                                 const bsa_tensor *seqused, const bsa_tensor *bt,
                                 const bsa_params *prm, const bsa_tensor *dq,
                                 const bsa_tensor *dk, const bsa_tensor *dv,
                                 size_t *workspace_bytes) {
  if (!workspace_bytes) return BSA_ERR_NULLPTR;
  bsa_ws_layout l;
  bsa_status st = bsa_bwd_workspace_layout(q, k, v, out, dout, lse, index, cu_q, cu_kv, seqused,
                                           bt, prm, dq, dk, dv, &l);
  if (st == BSA_OK) *workspace_bytes = size_t(l.total_bytes);
  return st;
}

bsa_status bsa_bwd(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                   const bsa_tensor *out, const bsa_tensor *dout, const bsa_tensor *lse,
                   const bsa_tensor *index, const bsa_tensor *cu_q, const bsa_tensor *cu_kv,
                   const bsa_tensor *seqused, const bsa_tensor *bt, const bsa_params *prm,
                   const bsa_tensor *dq, const bsa_tensor *dk, const bsa_tensor *dv,
                   void *workspace, size_t workspace_bytes, void *stream) {
  cudaEvent_t e0, e1;
  take_events(e0, e1);
  Problem p;
  Layout L;
  bool empty;
  bsa_status st = prepare(bwd_args(q, k, v, out, dout, lse, index, cu_q, cu_kv, seqused, bt, prm,
                                   dq, dk, dv), p, L, empty);
  if (st != BSA_OK || empty) return st;
  if ((st = check_ws(L, workspace, workspace_bytes)) != BSA_OK) return st;
  carve(p, L, workspace);
  return run_bwd(p, static_cast<cudaStream_t>(stream), e0, e1);
}

bsa_status bsa_read_status(const void *workspace, void *stream, uint32_t *flags) {
  if (!workspace || !flags) return BSA_ERR_NULLPTR;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ERR_CUDA;
  *flags = host;
  return BSA_OK;
}

}  // extern "C"
