// tma_maps.cu -- encodes the TMA tensor maps of one call (host side).  The
// driver's cuTensorMapEncodeTiled is reached through the runtime's
// entry-point query, so the library needs no link-time libcuda.
#include <cuda.h>
#include <cstring>
#include <cuda_runtime.h>

#include <mutex>

#include "tc_common.h"

namespace bsa {
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                 const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                 const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(f);
  });
  return fn;
}

// bytes per element of q / k / v
int64_t esz(const Problem &p) { return p.dtype == BSA_F8E4M3 ? 1 : 2; }

// Tiles of 128-byte rows: 5-D {128-byte column groups (64 16-bit or 128
// 8-bit columns), rows, D*esz/128 groups, heads, batch or page}; one box
// {128/esz, 128, D*esz/128, 1, 1} lands as consecutive 128-row x 128-byte
// boxes (16 KB each, 128-byte swizzle), i.e. a whole 128-row tile in one copy.
cudaError_t encode(CUtensorMap *m, const Problem &p, const void *base, const cuuint64_t dims[5],
                   const cuuint64_t strides[4], const cuuint32_t *box_in = nullptr) {
  EncodeTiled fn = encoder();
  if (!fn) return cudaErrorNotSupported;
  const cuuint32_t box_tile[5] = {cuuint32_t(128 / esz(p)), 128, cuuint32_t(p.D * esz(p) / 128), 1, 1};
  const cuuint32_t *box = box_in ? box_in : box_tile;
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUtensorMapDataType dt = p.dtype == BSA_F8E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : p.dtype == BSA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = fn(m, dt, 5, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t dq_acc_map(CUtensorMap *m, const Problem &p) {
  EncodeTiled fn = encoder();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {cuuint64_t(p.D), cuuint64_t(p.N1), cuuint64_t(p.rows_q)};
  const cuuint64_t strides[2] = {cuuint64_t(p.D) * 4, cuuint64_t(p.N1) * p.D * 4};
  const cuuint32_t box[3] = {32, 1, 128};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.dq_acc, dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cuuint64_t nz(int64_t x) { return x > 0 ? cuuint64_t(x) : 16; }

cudaError_t kv_map(CUtensorMap *m, const Problem &p, const void *base, int64_t sb, int64_t sh,
                   int64_t st) {
  const int64_t e = esz(p);
  const cuuint64_t inner = cuuint64_t(128 / e), halves = cuuint64_t(p.D * e / 128);
  if (p.kv_layout == BSA_LAYOUT_PA_BBND) {
    // {128 B, page rows, groups, kv heads, pages}
    const cuuint64_t dims[5] = {inner, cuuint64_t(p.page_size), halves, cuuint64_t(p.N2), cuuint64_t(p.num_pages)};
    const cuuint64_t strides[4] = {nz(st * e), 128, nz(sh * e), nz(sb * e)};
    return encode(m, p, base, dims, strides);
  }
  // {128 B, token rows, groups, kv heads, batch}
  const int64_t rows = p.kv_layout == BSA_LAYOUT_TND ? p.Tkv : p.Skv;
  const int64_t nb = p.kv_layout == BSA_LAYOUT_TND ? 1 : p.B;
  const cuuint64_t dims[5] = {inner, cuuint64_t(rows), halves, cuuint64_t(p.N2), cuuint64_t(nb)};
  const cuuint64_t strides[4] = {nz(st * e), 128, nz(sh * e),
                                 nz(p.kv_layout == BSA_LAYOUT_TND ? rows * st * e : sb * e)};
  return encode(m, p, base, dims, strides);
}

cudaError_t q_map(CUtensorMap *m, const Problem &p, const void *base, int64_t sb, int64_t sh,
                  int64_t st) {
  // {128 B, token rows, groups, q heads, batch}
  const int64_t e = esz(p);
  const int64_t rows = p.q_layout == BSA_LAYOUT_TND ? p.Tq : p.Sq;
  const int64_t nb = p.q_layout == BSA_LAYOUT_TND ? 1 : p.B;
  const cuuint64_t dims[5] = {cuuint64_t(128 / e), cuuint64_t(rows), cuuint64_t(p.D * e / 128), cuuint64_t(p.N1),
                              cuuint64_t(nb)};
  const cuuint64_t strides[4] = {nz(st * e), 128, nz(sh * e),
                                 nz(p.q_layout == BSA_LAYOUT_TND ? rows * st * e : sb * e)};
  return encode(m, p, base, dims, strides);
}

// Packed-head query tiles: {128 B, token rows, q heads, groups, batch} with
// box {128 B, 128/g, g, groups, 1}: the copy lands group by group, each group
// head-major (g heads x 128/g rows of 128 bytes), i.e. one 128-row tile whose
// row r is query row r % (128/g) of head r / (128/g).
cudaError_t q_map_packed(CUtensorMap *m, const Problem &p) {
  const int64_t e = esz(p);
  const int64_t rows = p.q_layout == BSA_LAYOUT_TND ? p.Tq : p.Sq;
  const int64_t nb = p.q_layout == BSA_LAYOUT_TND ? 1 : p.B;
  const cuuint64_t dims[5] = {cuuint64_t(128 / e), cuuint64_t(rows), cuuint64_t(p.N1),
                              cuuint64_t(p.D * e / 128), cuuint64_t(nb)};
  const cuuint64_t strides[4] = {nz(p.q_st * e), nz(p.q_sh * e), 128,
                                 nz(p.q_layout == BSA_LAYOUT_TND ? rows * p.q_st * e : p.q_sb * e)};
  const cuuint32_t box[5] = {cuuint32_t(128 / e), cuuint32_t(128 / p.pack_g), cuuint32_t(p.pack_g),
                             cuuint32_t(p.D * e / 128), 1};
  return encode(m, p, p.q, dims, strides, box);
}

}  // namespace

cudaError_t make_fwd_maps(const Problem &p, FwdMaps &m) {
  cudaError_t e = p.pack_g > 1 ? q_map_packed(&m.q, p) : q_map(&m.q, p, p.q, p.q_sb, p.q_sh, p.q_st);
  if (e != cudaSuccess) return e;
  if ((e = kv_map(&m.k, p, p.k, p.k_sb, p.k_sh, p.k_st)) != cudaSuccess) return e;
  return kv_map(&m.v, p, p.v, p.v_sb, p.v_sh, p.v_st);
}

cudaError_t make_bwd_maps(const Problem &p, BwdMaps &m) {
  cudaError_t e = q_map(&m.q, p, p.q, p.q_sb, p.q_sh, p.q_st);
  if (e != cudaSuccess) return e;
  if ((e = q_map(&m.dout, p, p.dout, p.do_sb, p.do_sh, p.do_st)) != cudaSuccess) return e;
  if ((e = kv_map(&m.k, p, p.k, p.k_sb, p.k_sh, p.k_st)) != cudaSuccess) return e;
  if ((e = kv_map(&m.v, p, p.v, p.v_sb, p.v_sh, p.v_st)) != cudaSuccess) return e;
  if (!p.dq_acc) {  // deterministic backward: no accumulator, the map is never used
    std::memset(&m.dq_acc, 0, sizeof(m.dq_acc));
    return cudaSuccess;
  }
  return dq_acc_map(&m.dq_acc, p);
}

cudaError_t make_dq_maps(const Problem &p, DqMaps &m) {
  cudaError_t e = q_map(&m.q, p, p.q, p.q_sb, p.q_sh, p.q_st);
  if (e != cudaSuccess) return e;
  if ((e = q_map(&m.dout, p, p.dout, p.do_sb, p.do_sh, p.do_st)) != cudaSuccess) return e;
  if ((e = kv_map(&m.k, p, p.k, p.k_sb, p.k_sh, p.k_st)) != cudaSuccess) return e;
  return kv_map(&m.v, p, p.v, p.v_sb, p.v_sh, p.v_st);
}

}  // namespace bsa
