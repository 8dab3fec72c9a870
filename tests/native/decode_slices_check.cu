// Host-side check of the tensor-core decode's work division
// (latent_attention_b200/csrc/decode_slices.cuh, the code both decode kernels
// run): over many random batches, every token of every valid sequence lies in
// exactly one unit's segment; a segment is "whole" exactly when one unit holds
// the sequence; the partial slots of a sequence's units are the ones the
// combine kernel reads, distinct and inside the unit's two slots; the
// per-unit cursor visits exactly the non-empty segments in order.
// Prints "ok <cases>" or the first violation (exit status 1).
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <random>
#include <set>
#include <vector>

#include "decode_slices.cuh"

using namespace mla::slices;

static int fail(const char* what, int c, int b, int u) {
  std::printf("FAIL case %d seq %d unit %d: %s\n", c, b, u, what);
  return 1;
}

int main() {
  std::mt19937 rng(12345);
  int cases = 0;
  for (int c = 0; c < 3000; ++c) {
    // batch shapes: few long sequences, many short ones, mixes, empties
    const int kind = c % 5;
    const int B = kind == 0 ? 1 + (int)(rng() % 4) : kind == 1 ? 200 + (int)(rng() % 400)
                                                   : 1 + (int)(rng() % 80);
    const int max_ctx = kind == 0 ? 70000 : kind == 1 ? 16 : 1 + (int)(rng() % 40000);
    std::vector<int32_t> cu(B + 1);
    cu[0] = (int32_t)(rng() % 3);      // a non-zero base offset is allowed
    std::vector<int> n(B);
    for (int b = 0; b < B; ++b) {
      int len = 1 + (int)(rng() % max_ctx);
      if (kind == 4 && rng() % 7 == 0) len = 0;                 // invalid: empty
      if (kind == 4 && rng() % 11 == 0) len = max_ctx + 1;      // invalid: too long
      n[b] = len;
      cu[b + 1] = cu[b] + len;
    }
    const int n_units = 1 + (int)(rng() % 74);
    const int min_len = (c % 3 == 0) ? 512 : 1 + (int)(rng() % 2048);

    // D2's view: each unit's segments
    std::vector<std::vector<std::pair<int, int>>> cover(B);   // [t0, t0 + tcount)
    std::map<int, std::set<int>> units_of;                      // seq -> units with tokens
    std::map<std::pair<int, int>, int> slot_of;                 // (seq, unit) -> slot
    std::map<std::pair<int, int>, bool> whole_of;
    std::set<int> used_slots;
    for (int u = 0; u < n_units; ++u) {
      const Slice sl = unit_slice(cu.data(), B, max_ctx, u, n_units, min_len);
      if (sl.r0 >= sl.r1) continue;
      const int b0 = seq_at(cu.data(), B, sl.r0), b1 = seq_at(cu.data(), B, sl.r1 - 1) + 1;
      std::vector<int> nonempty;
      for (int b = b0; b < b1; ++b) {
        const Seg s = seg_info(cu.data(), b, max_ctx, sl, u);
        if (s.nch == 0) continue;
        nonempty.push_back(b);
        if (s.tcount < 1 || s.t0 < 0 || s.t0 + s.tcount > n[b]) return fail("range", c, b, u);
        if (s.nch != (s.tcount + NT - 1) / NT) return fail("chunks", c, b, u);
        cover[b].push_back({s.t0, s.t0 + s.tcount});
        units_of[b].insert(u);
        slot_of[{b, u}] = s.slot;
        whole_of[{b, u}] = s.whole;
        if (s.slot != 2 * u && s.slot != 2 * u + 1) return fail("slot range", c, b, u);
        if (!s.whole && !used_slots.insert(s.slot).second) return fail("slot reused", c, b, u);
      }
      // the cursor walks exactly the non-empty segments, chunk by chunk
      SegCursor cur;
      cur.start(cu.data(), b0, b1, max_ctx, sl, u);
      size_t seen = 0;
      int kk = 0;
      while (!cur.done) {
        if (seen >= nonempty.size() || cur.s.b != nonempty[seen] || cur.kk != kk)
          return fail("cursor order", c, cur.s.b, u);
        const int nch = cur.s.nch;
        for (int j = 1; j < nch; ++j)
          if (cur.next(cu.data(), b0, b1, max_ctx, sl, u)) return fail("cursor chunks", c, cur.s.b, u);
        cur.next(cu.data(), b0, b1, max_ctx, sl, u);
        ++seen;
        ++kk;
      }
      if (seen != nonempty.size()) return fail("cursor count", c, -1, u);
    }
    // every valid sequence covered exactly once; the combine's view agrees
    for (int b = 0; b < B; ++b) {
      const bool valid = n[b] >= 1 && n[b] <= max_ctx;
      const SeqUnits su = seq_units(cu.data(), b, B, max_ctx, n_units, min_len);
      if (!valid) {
        if (!cover[b].empty()) return fail("invalid sequence has segments", c, b, -1);
        if (su.valid) return fail("invalid sequence accepted by combine", c, b, -1);
        continue;
      }
      // An over-long sequence can push the stream past B max_ctx tokens; the
      // sequences beyond that bound are refused (and reported) as a whole.
      const int64_t Tt = stream_tokens(cu.data(), B, max_ctx);
      if ((int64_t)cu[b + 1] - cu[0] > Tt) {
        if (su.valid) return fail("sequence past the stream accepted", c, b, -1);
        continue;
      }
      if (!su.valid) return fail("valid sequence refused by combine", c, b, -1);
      auto v = cover[b];
      std::sort(v.begin(), v.end());
      int64_t at = 0;
      for (auto& iv : v) {
        if (iv.first != at) return fail("gap or overlap", c, b, -1);
        at = iv.second;
      }
      if (at != n[b]) return fail("not covered", c, b, -1);
      const std::set<int>& us = units_of[b];
      if ((int)us.size() != su.u1 - su.u0 + 1 || *us.begin() != su.u0 || *us.rbegin() != su.u1)
        return fail("units differ from the combine's", c, b, -1);
      for (int u : us) {
        if (whole_of[{b, u}] != (su.u0 == su.u1)) return fail("whole flag", c, b, u);
        if (su.u0 != su.u1 && slot_of[{b, u}] != seq_slot(su, u)) return fail("slot differs", c, b, u);
      }
    }
    ++cases;
  }
  std::printf("ok %d\n", cases);
  return 0;
}
