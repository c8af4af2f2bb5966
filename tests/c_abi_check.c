/* A plain C caller of libbsa.so: compiled with gcc against include/bsa.h
 * alone (no torch, no Python), it sizes a forward and a backward workspace
 * and checks a few host-side refusals.  Only host validation runs here, so
 * the tensor pointers are stand-in addresses that are never dereferenced.
 * Prints "ok" and returns 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "bsa.h"

static bsa_tensor dense(uintptr_t addr, int32_t dtype, int ndim, const int64_t *shape) {
  bsa_tensor t;
  memset(&t, 0, sizeof(t));
  t.data = (void *)addr;
  t.dtype = dtype;
  t.ndim = ndim;
  int64_t st = 1;
  for (int i = ndim - 1; i >= 0; --i) {
    t.shape[i] = shape[i];
    t.stride[i] = st;
    st *= shape[i];
  }
  return t;
}

#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                      \
    }                                                                \
  } while (0)

int main(void) {
  CHECK(bsa_abi_version() == 3);
  CHECK(strncmp(bsa_status_string(BSA_ERR_WORKSPACE), "BSA_ERR_WORKSPACE", 17) == 0);

  /* BNSD B=1, N1=4 query heads over N2=2 kv heads, S=512, D=128, blocks (128,128) */
  const int64_t qs[4] = {1, 4, 512, 128}, ks[4] = {1, 2, 512, 128};
  const int64_t is[4] = {1, 4, 4, 4}, ls[3] = {1, 4, 512};
  bsa_tensor q = dense(0x100000, BSA_BF16, 4, qs), k = dense(0x200000, BSA_BF16, 4, ks);
  bsa_tensor v = dense(0x300000, BSA_BF16, 4, ks), out = dense(0x400000, BSA_BF16, 4, qs);
  bsa_tensor idx = dense(0x500000, BSA_U16, 4, is), lse = dense(0x600000, BSA_F32, 3, ls);
  bsa_tensor dout = dense(0x700000, BSA_BF16, 4, qs), dq = dense(0x800000, BSA_BF16, 4, qs);
  bsa_tensor dk = dense(0x900000, BSA_BF16, 4, ks), dv = dense(0xA00000, BSA_BF16, 4, ks);

  bsa_params P;
  memset(&P, 0, sizeof(P));
  P.q_layout = BSA_LAYOUT_BNSD;
  P.kv_layout = BSA_LAYOUT_BNSD;
  P.num_heads = 4;
  P.num_kv_heads = 2;
  P.block_shape[0] = 128;
  P.block_shape[1] = 128;
  P.return_lse = 1;
  P.mask_type = BSA_MASK_CAUSAL;

  size_t nf = 0, nb = 0, nd = 0;
  CHECK(bsa_fwd_get_workspace(&q, &k, &v, &idx, NULL, NULL, NULL, NULL, &P, &out, &lse, &nf) == BSA_OK);
  CHECK(nf > 0 && nf % 256 == 0);
  CHECK(bsa_bwd_get_workspace(&q, &k, &v, &out, &dout, &lse, &idx, NULL, NULL, NULL, NULL, &P, &dq,
                              &dk, &dv, &nb) == BSA_OK);
  P.deterministic = 1;
  CHECK(bsa_bwd_get_workspace(&q, &k, &v, &out, &dout, &lse, &idx, NULL, NULL, NULL, NULL, &P, &dq,
                              &dk, &dv, &nd) == BSA_OK);
  CHECK(nb > nd); /* the deterministic backward has no fp32 dQ accumulator */

  /* refusals: 3 query heads over 2 kv heads; a missing index; a too-small workspace */
  P.num_heads = 3;
  CHECK(bsa_fwd_get_workspace(&q, &k, &v, &idx, NULL, NULL, NULL, NULL, &P, &out, &lse, &nf) ==
        BSA_ERR_PARAM_INVALID);
  P.num_heads = 4;
  CHECK(bsa_fwd_get_workspace(&q, &k, &v, NULL, NULL, NULL, NULL, NULL, &P, &out, &lse, &nf) ==
        BSA_ERR_NULLPTR);
  CHECK(bsa_fwd(&q, &k, &v, &idx, NULL, NULL, NULL, NULL, &P, &out, &lse, (void *)0xB00000, 256,
                NULL) == BSA_ERR_WORKSPACE);
  printf("ok\n");
  return 0;
}
