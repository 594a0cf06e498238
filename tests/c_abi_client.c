/* A plain C client of libmedusa.so: calls the host-only entry points
 * through include/medusa.h (no CUDA call) and prints the tree plan of
 * (K, s, N) one node per line as "parent depth r_1 .. r_K", then the first
 * ancestor-mask word of every node.  Used by tests/test_c_abi.py. */
#include <stdio.h>
#include <stdlib.h>

#include "medusa.h"

int main(int argc, char** argv) {
  if (argc != 4) {
    fprintf(stderr, "usage: %s K s N\n", argv[0]);
    return 2;
  }
  const int K = atoi(argv[1]), s = atoi(argv[2]), N = atoi(argv[3]);
  const int W = (N + 31) / 32;
  int32_t* parent = malloc(sizeof(int32_t) * (size_t)N);
  int32_t* depth = malloc(sizeof(int32_t) * (size_t)N);
  int32_t* rank = malloc(sizeof(int32_t) * (size_t)N * (size_t)K);
  uint32_t* anc = malloc(sizeof(uint32_t) * (size_t)N * (size_t)W);
  if (!parent || !depth || !rank || !anc) return 3;
  const int rc = medusa_tree_plan_host(K, s, N, parent, depth, rank, anc);
  printf("version %s\n", medusa_version());
  printf("status %d\n", rc);
  if (rc != MEDUSA_OK) {
    printf("error %s\n", medusa_last_error());
    return 0;
  }
  for (int n = 0; n < N; ++n) {
    printf("%d %d", parent[n], depth[n]);
    for (int k = 0; k < K; ++k) printf(" %d", rank[(size_t)n * K + k]);
    printf(" %u\n", anc[(size_t)n * W]);
  }
  free(parent);
  free(depth);
  free(rank);
  free(anc);
  return 0;
}
