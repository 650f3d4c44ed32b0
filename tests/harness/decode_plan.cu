// Host build of the Phase-2 work planning (star_plan.h) for CPU tests: the
// same functions the C ABI calls, exported with C linkage.
#include "star_plan.h"

extern "C" {

int dp_decode_chunk(int B, int Hkv, int L, int b, int tail_plus_T, int sms) {
  const int n = star::ceil_div(L, b);
  return star::decode_chunk(B, Hkv, L, b, n, n + 1, tail_plus_T, sms);
}

int dp_chunks_per_head(int L, int b, int tail_plus_T, int chunk, int* nc3) {
  const int n = star::ceil_div(L, b);
  return star::decode_chunks_per_head(L, b, n, tail_plus_T, chunk, &nc3[0], &nc3[1], &nc3[2]);
}

long long dp_units_bound(int B, int Hkv, int Lcap, int b) {
  return star::decode_units_bound(B, Hkv, Lcap, b);
}

int dp_max_chunks_per_split() { return star::kMaxChunksPerSplit; }
int dp_tile() { return star::kDecTile; }

}  // extern "C"
