/* A plain C consumer of libnattn: host-side entry points only (no GPU).
 * Prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "nattn.h"

static int fails = 0;
#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "check failed: %s (line %d)\n", #c, __LINE__); \
      ++fails;                                                     \
    }                                                              \
  } while (0)

static void dense_args(nattn_args* a, int normalizer) {
  memset(a, 0, sizeof(*a));
  /* pointers are not dereferenced by the size query or by validation */
  a->q = a->k = a->v = (const void*)0x1000;
  a->out = (void*)0x1000;
  a->B = 1; a->Hq = 4; a->Hkv = 2; a->Tq = 256; a->Tk = 256; a->d = 128; a->dv = 128;
  a->scale = 0.088388f;
  a->normalizer = normalizer;
  a->causal = 1;
}

int main(void) {
  nattn_args a;
  CHECK(nattn_version() > 0);
  CHECK(strcmp(nattn_strerror(NATTN_OK), "ok") == 0);
  CHECK(strlen(nattn_strerror(NATTN_ETIMEOUT)) > 0);

  /* softmax prefill needs no scratch; the sparse normalizers do */
  dense_args(&a, NATTN_SOFTMAX);
  CHECK(nattn_workspace_size(&a) == 0);
  dense_args(&a, NATTN_SPARSEMAX);
  const size_t ws = nattn_workspace_size(&a);
  CHECK(ws > 0);

  /* scratch smaller than asked for is refused before any launch */
  a.workspace = (void*)0x1000;
  a.workspace_bytes = ws - 1;
  CHECK(nattn_fwd_ex(&a) == NATTN_EWORKSPACE);

  /* invalid argument blocks are refused before any launch */
  dense_args(&a, NATTN_SOFTMAX);
  a.Hkv = 3;  /* Hq % Hkv != 0 */
  CHECK(nattn_fwd_ex(&a) == NATTN_EINVAL);
  dense_args(&a, 7);  /* no such normalizer */
  CHECK(nattn_fwd_ex(&a) == NATTN_EINVAL);
  CHECK(nattn_fwd_ex(NULL) == NATTN_EINVAL);

  if (fails == 0) printf("ok\n");
  return fails == 0 ? 0 : 1;
}
