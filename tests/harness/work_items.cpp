// Host build of the attention kernels' work decomposition (star_index.cuh),
// for CPU tests: the same header the kernels include, with the CUDA function
// qualifiers defined away. Each call builds the geometry the way the
// library's entry points do (hpc = 2 query-head tiles per item when the GQA
// group size is even, else 1; two heads per tile for query chunks of at most
// 64 tokens when the group has 4 or more heads) and writes one work item as
// 8 + 2 * 6 integers:
// b, kvh, slot0, q_lo, q_hi, pos_base, split, nspan, then per span key0,
// ntiles, lo, hi, causal, src.
#define __host__
#define __device__
#define __forceinline__ inline
#include "star_index.cuh"

using star::AttnGeom;
using star::WorkItem;

static AttnGeom geom(int B, int Hq, int Hkv, int L, int b, int a) {
  AttnGeom g{};
  g.B = B;
  g.Hq = Hq;
  g.Hkv = Hkv;
  g.hpc = ((Hq / Hkv) % 2 == 0) ? 2 : 1;
  g.hps = 1;
  g.L = L;
  g.b = b;
  g.a = a;
  g.n = star::ceil_div(L, b);
  return g;
}

static void put(const WorkItem& w, int* out) {
  const int head[8] = {w.b, w.kvh, w.slot0, w.q_lo, w.q_hi, w.pos_base, w.split, w.nspan};
  for (int i = 0; i < 8; ++i) out[i] = head[i];
  for (int s = 0; s < 2; ++s) {
    const star::KvSpan& sp = w.span[s];
    const int v[6] = {sp.key0, sp.ntiles, sp.lo, sp.hi, sp.causal, sp.src};
    for (int i = 0; i < 6; ++i) out[8 + 6 * s + i] = v[i];
  }
}

extern "C" {

int wi_hpc(int Hq, int Hkv) { return ((Hq / Hkv) % 2 == 0) ? 2 : 1; }

// query heads per Phase-2 item (two tiles of two heads for chunks of <= 64 tokens)
int wi_phase2_heads_per_item(int Hq, int Hkv, int T) {
  return wi_hpc(Hq, Hkv) * star::chunk_heads_per_slot(T, Hq, Hkv);
}

int wi_phase1_items(int B, int Hq, int Hkv, int L, int b, int a) {
  return geom(B, Hq, Hkv, L, b, a).phase1_items();
}

void wi_phase1_item(int B, int Hq, int Hkv, int L, int b, int a, int item, int* out) {
  put(geom(B, Hq, Hkv, L, b, a).phase1_item(item), out);
}

static AttnGeom geom2(int B, int Hq, int Hkv, int L, int b, int T, int tail_len, int with_tail,
                      int nsub) {
  AttnGeom g = geom(B, Hq, Hkv, L, b, 0);
  g.hps = star::chunk_heads_per_slot(T, Hq, Hkv);
  g.T = T;
  g.tail_len = tail_len;
  g.tail = with_tail;
  g.nsub = nsub;
  g.sub_len = b / nsub;
  return g;
}

int wi_phase2_items(int B, int Hq, int Hkv, int L, int b, int T, int tail_len, int with_tail,
                    int nsub) {
  return geom2(B, Hq, Hkv, L, b, T, tail_len, with_tail, nsub).phase2_items();
}

int wi_phase2_splits(int B, int Hq, int Hkv, int L, int b, int T, int tail_len, int with_tail,
                     int nsub) {
  return geom2(B, Hq, Hkv, L, b, T, tail_len, with_tail, nsub).phase2_splits();
}

void wi_phase2_item(int B, int Hq, int Hkv, int L, int b, int T, int tail_len, int with_tail,
                    int nsub, int item, int* out) {
  put(geom2(B, Hq, Hkv, L, b, T, tail_len, with_tail, nsub).phase2_item(item), out);
}

}  // extern "C"
