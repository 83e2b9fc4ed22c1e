// Row geometry shared by the sparse-MLA kernels: where a query row's keys live
// in the latent cache, how many it may see, and how long its key list is.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsa {

struct RowGeom {
  int64_t kbase, nvis, n_list;
  int64_t klen;  // keys the row's sequence holds (the bound of MTP's extra keys)
};

// Where the row's keys live and how many it sees, from the caller's inputs alone
// (not the index list): clamped, and flagged by one thread. n_list = nvis.
__device__ __forceinline__ RowGeom row_base(const MlaArgs& a, int r, bool report);

// The list of a row whose index list came from the top-k (forced columns first):
// the expected length L, its known prefix K (the forced columns, or the whole
// list of a dense row) and the key of a known slot, all from the position.
// ext: keys after the row's own position that it also attends to (an MTP draft
// step's newer keys, nvis .. nvis+ext-1); they follow the list.
struct ListPlan {
  int64_t L, K;
  int64_t hi;    // first local-window column (non-dense rows)
  int64_t nvis;
  int ext;
  bool dense;
};
__device__ __forceinline__ ListPlan list_plan(const MlaArgs& a, int64_t nvis, int ext = 0) {
  ListPlan p;
  p.dense = nvis <= a.topk;
  p.L = min64(nvis, (int64_t)a.topk);
  p.K = p.dense ? p.L : min64(p.L, (int64_t)a.n_init + a.n_loc);
  p.hi = nvis - a.n_loc;
  p.nvis = nvis;
  p.ext = ext;
  return p;
}
__device__ __forceinline__ int64_t known_key(const ListPlan& p, const MlaArgs& a, int64_t i) {
  return (p.dense || i < a.n_init) ? i : p.hi + (i - a.n_init);
}

// A split's tiles (kTK keys each) of a forced-first list: whole tiles of the known prefix,
// then whole tiles of the rest read from the list, each part shared evenly by
// the splits. The known prefix is the forced columns' whole tiles (a dense
// row: its whole list); the forced columns left over in a part tile are read
// from the list with the selected ones, which the top-k wrote in the same
// order, so a sparse row of 2048 keys is 64 full tiles (1024 + 1024 keys), not
// 65 with two part tiles. ub = the first slot read from the list.
// An MTP draft step's newer keys (p.ext of them) are known as well: a dense
// row's known run simply continues past its position; a sparse row gets one
// more known tile after its forced ones.
struct FfTiles {
  int kt0, kt, ut0, ut;
  int64_t ub;
  int kf;  // known tiles holding forced (or dense) keys; a known tile kf holds the extra keys
};
template <int kTK>
__device__ __forceinline__ FfTiles ff_tiles(const ListPlan& p, int s, int n) {
  FfTiles f;
  f.kf = (int)(p.dense ? (p.K + p.ext + kTK - 1) / kTK : p.K / kTK);
  const int Kt = f.kf + (!p.dense && p.ext > 0 ? 1 : 0);
  f.ub = min64((int64_t)f.kf * kTK, p.L);
  const int Ut = (int)((p.L - f.ub + kTK - 1) / kTK);
  f.kt0 = Kt * s / n;
  f.kt = Kt * (s + 1) / n - f.kt0;
  f.ut0 = Ut * s / n;
  f.ut = Ut * (s + 1) / n - f.ut0;
  return f;
}
// The key of known slot sl (-1: masked).
template <int kTK>
__device__ __forceinline__ int known_slot_key(const ListPlan& p, const FfTiles& f, const MlaArgs& a, int64_t sl) {
  if (p.dense) return sl < p.K + p.ext ? (int)sl : -1;
  if (sl < (int64_t)f.kf * kTK) return sl < p.K ? (int)known_key(p, a, sl) : -1;
  const int64_t e = sl - (int64_t)f.kf * kTK;
  return e < p.ext ? (int)(p.nvis + e) : -1;
}
// Extra keys of sub-block z of an MTP launch, clipped to the sequence (flagged).
__device__ __forceinline__ int mtp_ext(const MlaArgs& a, const RowGeom& g, int z, bool report) {
  if (!a.mtp || g.nvis <= 0) return 0;
  int e = z;
  if (g.nvis + e > g.klen) {
    if (report) flag_error(a.err, LSA_DEVERR_POS);
    e = (int)max64(0, g.klen - g.nvis);
  }
  return e;
}

// A LoZA row that sees nvis keys ("LongCat-Flash-Thinking-ZigZag架构深度剖析",
// "稀疏模式设计": Sink, Recent and Chunked regions): its keys are [0, s_end) and
// [w0, nvis), w0 the earlier of the recent window's and the own chunk's first
// key (never inside the sink run). Slot i holds key i below s_end, else
// w0 + (i - s_end).
struct LozaSpan {
  int64_t s_end, w0;
};
__device__ __forceinline__ LozaSpan loza_span(const MlaArgs& a, int64_t nvis) {
  const int64_t p = nvis - 1;
  LozaSpan z;
  z.s_end = min64((int64_t)a.loza_sink, nvis);
  z.w0 = max64(min64(p - a.loza_recent + 1, (p / a.loza_chunk) * a.loza_chunk), z.s_end);
  return z;
}
__device__ __forceinline__ int64_t loza_key(const LozaSpan& z, int64_t i) { return i < z.s_end ? i : z.w0 + (i - z.s_end); }

// Row geometry, with every out-of-range input clamped (and flagged by one thread).
__device__ __forceinline__ RowGeom row_geometry(const MlaArgs& a, int r, bool report) {
  RowGeom g{0, 0, 0, 0};
  if (a.decode) {
    const int seq = a.seq_of_row ? a.seq_of_row[r] : r;
    if (seq < 0 || seq >= a.n_seq) {
      if (report) flag_error(a.err, LSA_DEVERR_SEQ);
    } else {
      g.kbase = a.k_off[seq];
      const int64_t klen = a.k_off[seq + 1] - g.kbase;
      g.klen = klen;
      g.nvis = klen;
      if (a.pos) {
        int64_t p1 = (int64_t)a.pos[r] + 1;
        if (p1 < 1 || p1 > klen) {
          if (report) flag_error(a.err, LSA_DEVERR_POS);
          p1 = max64(0, min64(p1, klen));
        }
        g.nvis = p1;
      }
    }
  } else {
    g.klen = a.n_keys;
    int64_t p1 = (int64_t)a.pos[r] + 1;
    if (p1 < 1 || p1 > a.n_keys) {
      if (report) flag_error(a.err, LSA_DEVERR_POS);
      p1 = max64(0, min64(p1, a.n_keys));
    }
    g.nvis = p1;
  }
  g.n_list = g.nvis;
  if (a.loza && g.nvis > 0) {
    const LozaSpan z = loza_span(a, g.nvis);
    g.n_list = z.s_end + g.nvis - z.w0;
  }
  if (a.idx) {
    int c = a.count[r];
    if (c < 0 || c > a.topk) {
      if (report) flag_error(a.err, LSA_DEVERR_COUNT);
      c = max(0, min(c, a.topk));
    }
    g.n_list = c;
  }
  return g;
}

__device__ __forceinline__ RowGeom row_base(const MlaArgs& a, int r, bool report) {
  MlaArgs b = a;
  b.idx = nullptr;  // (row_geometry then reads no count)
  return row_geometry(b, r, report);
}

}  // namespace lsa
