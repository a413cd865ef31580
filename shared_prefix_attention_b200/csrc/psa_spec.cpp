// Host-side mask builder: segment forest -> visibility rectangles -> tile
// schedule.  "KV-0 redundancy prefix sharing attention mask design"
// (PrefixSharing PR #50): design summary (visibility from a block-causal
// rectangle spec, not a dense mask, prefix K/V stored once) and key changes
// section 2 (mask construction for the flat GRPO case and the multi-level
// tree / chain case).
#include <algorithm>
#include <cstdint>
#include <vector>

#include "psa.h"

namespace {

struct Range {
  int32_t a, b;  // [a, b)
};

// Visible pairs of rectangle r inside the box [qa,qb) x [ka,kb).
int64_t visible_in_box(const psa_rect& r, int32_t qa, int32_t qb, int32_t ka, int32_t kb) {
  int32_t q_lo = std::max(qa, r.q0), q_hi = std::min(qb, r.q1);
  int32_t k_lo = std::max(ka, r.k0), k_hi = std::min(kb, r.k1);
  if (q_lo >= q_hi || k_lo >= k_hi) return 0;
  if (!r.causal) return int64_t(q_hi - q_lo) * (k_hi - k_lo);
  int64_t n = 0;
  for (int32_t q = q_lo; q < q_hi; ++q) {
    if (r.causal == 1) {
      // causal: k - k0 <= q - q0
      int32_t last = std::min<int32_t>(k_hi - 1, r.k0 + (q - r.q0));
      if (last >= k_lo) n += last - k_lo + 1;
    } else {
      // transposed causal (keys as rows): k - k0 >= q - q0
      int32_t first = std::max<int32_t>(k_lo, r.k0 + (q - r.q0));
      if (first < k_hi) n += k_hi - first;
    }
  }
  return n;
}

}  // namespace

extern "C" int psa_spec_flat(int32_t P, int32_t N, int32_t S, psa_segment* out,
                             int32_t cap, int32_t* nout) {
  if (!nout || P < 0 || N < 0 || (N > 0 && S <= 0) || (P == 0 && N == 0))
    return PSA_ERR_INVALID_ARG;
  int32_t need = N + (P > 0 ? 1 : 0);
  *nout = need;
  if (cap < need || !out) return PSA_ERR_CAPACITY;
  int32_t i = 0;
  if (P > 0) out[i++] = psa_segment{P, -1};
  for (int32_t s = 0; s < N; ++s) out[i++] = psa_segment{S, P > 0 ? 0 : -1};
  return PSA_OK;
}

extern "C" int psa_build_spec(const psa_segment* segs, int32_t nseg, psa_rect* out,
                              int32_t cap, int32_t* nout) {
  if (!nout || nseg < 0 || (nseg > 0 && !segs)) return PSA_ERR_INVALID_ARG;
  std::vector<Range> flat(nseg);
  int64_t pos = 0;
  for (int32_t s = 0; s < nseg; ++s) {
    if (segs[s].len <= 0) return PSA_ERR_INVALID_ARG;
    if (segs[s].parent >= s || segs[s].parent < -1) return PSA_ERR_INVALID_ARG;
    if (pos + segs[s].len > INT32_MAX) return PSA_ERR_INVALID_ARG;
    flat[s] = Range{int32_t(pos), int32_t(pos + segs[s].len)};
    pos += segs[s].len;
  }
  // One causal rectangle per segment (itself) and one full rectangle per
  // (segment, ancestor) pair.  Ancestors precede in flat order, so every
  // key of an ancestor rectangle lies before every query of the segment.
  int64_t count = 0;
  for (int32_t s = 0; s < nseg; ++s)
    for (int32_t a = s; a >= 0; a = segs[a].parent) ++count;
  if (count > INT32_MAX) return PSA_ERR_INVALID_ARG;
  *nout = int32_t(count);
  if (cap < count || (count > 0 && !out)) return PSA_ERR_CAPACITY;
  int32_t i = 0;
  for (int32_t s = 0; s < nseg; ++s) {
    // ancestors first (root-most last visited -> emit in ascending key order)
    std::vector<int32_t> chain;
    for (int32_t a = segs[s].parent; a >= 0; a = segs[a].parent) chain.push_back(a);
    for (auto it = chain.rbegin(); it != chain.rend(); ++it)
      out[i++] = psa_rect{flat[s].a, flat[s].b, flat[*it].a, flat[*it].b, 0};
    out[i++] = psa_rect{flat[s].a, flat[s].b, flat[s].a, flat[s].b, 1};
  }
  return PSA_OK;
}

extern "C" int psa_transpose_spec(const psa_rect* rects, int32_t nrect, psa_rect* out) {
  if (nrect < 0 || (nrect > 0 && (!rects || !out))) return PSA_ERR_INVALID_ARG;
  for (int32_t r = 0; r < nrect; ++r) {
    const psa_rect x = rects[r];
    if (x.causal < 0 || x.causal > 2) return PSA_ERR_INVALID_ARG;
    // rows become keys and columns queries; a causal rectangle turns into
    // its transpose and back
    out[r] = psa_rect{x.k0, x.k1, x.q0, x.q1, x.causal == 0 ? 0 : 3 - x.causal};
  }
  return PSA_OK;
}

extern "C" int psa_build_schedule(const psa_rect* rects, int32_t nrect,
                                  const int32_t* cu_seqlens, int32_t ngroups, int32_t tile_m,
                                  int32_t tile_n, int32_t* out, int64_t cap, int64_t* nout) {
  if (!nout || nrect < 0 || (nrect > 0 && !rects) || !cu_seqlens || ngroups <= 0 ||
      tile_m <= 0 || (tile_m & 1) || tile_n <= 0)
    return PSA_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return PSA_ERR_INVALID_ARG;
  for (int32_t g = 0; g < ngroups; ++g)
    if (cu_seqlens[g + 1] <= cu_seqlens[g]) return PSA_ERR_INVALID_ARG;
  const int32_t T = cu_seqlens[ngroups];
  for (int32_t r = 0; r < nrect; ++r) {
    const psa_rect& x = rects[r];
    if (x.q0 < 0 || x.q1 > T || x.q0 >= x.q1 || x.k0 < 0 || x.k1 > T || x.k0 >= x.k1 ||
        x.causal < 0 || x.causal > 2)
      return PSA_ERR_INVALID_ARG;
  }
  const int32_t half = tile_m / 2;

  struct Item {
    int32_t q0, qlen, kv_begin, kv_count;
  };
  struct Kv {
    int32_t k0, klen, rb[2], rc[2], flags;
  };
  std::vector<Item> items;
  std::vector<Kv> kvs;
  std::vector<psa_rect> trects;
  std::vector<int32_t> cut;
  int32_t max_kv = 0;

  for (int32_t g = 0; g < ngroups; ++g) {
    const int32_t g0 = cu_seqlens[g], g1 = cu_seqlens[g + 1];
    std::vector<int32_t> grect;
    for (int32_t r = 0; r < nrect; ++r)
      if (rects[r].q0 < g1 && rects[r].q1 > g0) grect.push_back(r);
    for (int32_t qa = g0; qa < g1; qa += tile_m) {
      const int32_t qb = std::min(g1, qa + tile_m);
      Item it{qa, qb - qa, int32_t(kvs.size()), 0};
      for (int32_t ka = g0; ka < g1; ka += tile_n) {
        const int32_t kb = std::min(g1, ka + tile_n);
        Kv e{ka, kb - ka, {0, 0}, {0, 0}, 0};
        for (int h = 0; h < 2; ++h) {
          const int32_t ha = qa + h * half, hb = std::min(qb, ha + half);
          if (ha >= hb) continue;  // the block has no second half
          int64_t vis = 0;
          cut.clear();
          for (int32_t r : grect) {
            const int64_t n = visible_in_box(rects[r], ha, hb, ka, kb);
            if (n > 0) {
              vis += n;
              cut.push_back(r);
            }
          }
          if (vis == 0) continue;
          e.flags |= 1 << h;  // this half has visible pairs in the tile
          if (vis == int64_t(hb - ha) * (kb - ka)) {
            e.flags |= 4 << h;  // ... and all of them are visible
          } else {
            e.rb[h] = int32_t(trects.size());
            e.rc[h] = int32_t(cut.size());
            for (int32_t r : cut) trects.push_back(rects[r]);
          }
        }
        if (!e.flags) continue;
        kvs.push_back(e);
        ++it.kv_count;
      }
      max_kv = std::max(max_kv, it.kv_count);
      items.push_back(it);
    }
  }
  // longest-processing-time first; ties by position for determinism
  std::stable_sort(items.begin(), items.end(), [](const Item& a, const Item& b) {
    return a.kv_count > b.kv_count;
  });

  const int64_t need = 8 + 4 * int64_t(items.size()) + 8 * int64_t(kvs.size()) +
                       5 * int64_t(trects.size());
  *nout = need;
  if (need > INT32_MAX) return PSA_ERR_INVALID_ARG;
  if (cap < need || !out) return PSA_ERR_CAPACITY;
  out[0] = 0x50534132;
  out[1] = int32_t(items.size());
  out[2] = int32_t(kvs.size());
  out[3] = int32_t(trects.size());
  out[4] = tile_m;
  out[5] = tile_n;
  out[6] = T;
  out[7] = max_kv;
  int64_t o = 8;
  for (const Item& it : items) {
    out[o++] = it.q0;
    out[o++] = it.qlen;
    out[o++] = it.kv_begin;
    out[o++] = it.kv_count;
  }
  for (const Kv& e : kvs) {
    out[o++] = e.k0;
    out[o++] = e.klen;
    out[o++] = e.rb[0];
    out[o++] = e.rc[0];
    out[o++] = e.rb[1];
    out[o++] = e.rc[1];
    out[o++] = e.flags;
    out[o++] = 0;
  }
  for (const psa_rect& r : trects) {
    out[o++] = r.q0;
    out[o++] = r.q1;
    out[o++] = r.k0;
    out[o++] = r.k1;
    out[o++] = r.causal;
  }
  return PSA_OK;
}
