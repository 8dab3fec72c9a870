// How the tensor-core decode divides its work: the slices of the token
// stream, the segments inside a slice and the partial slots of the sequences
// that cross a slice boundary.  Host and device code, shared by the latent
// attention kernel, the combine kernel and a host-side check.
//
// The token stream of all sequences, concatenated in cu_ctx order, is cut
// into equal slices of L positions, one per CTA pair ("unit"); L is at least
// min_len.  Each sequence is charged kSeqCost positions ahead of its tokens
// (the cost of starting a segment: query loads, pipeline refill, epilogue,
// about 4.5 chunks), so a unit whose slice holds more sequence starts takes
// fewer tokens.  Sequence b occupies positions [vs_b, vs_b + kSeqCost + n_b)
// with vs_b = cu_ctx[b] - cu_ctx[0] + b kSeqCost.  A unit's segment of b is
// the part of b's tokens inside its slice.  A segment that covers all of b
// is written to o_lat directly; any other segment leaves a partial (o, lse)
// in slot 2u (the unit's first segment) or 2u + 1 (its last), which the
// combine kernel merges.
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define MLA_HD __host__ __device__ __forceinline__
#else
#define MLA_HD inline
#endif

namespace mla {
namespace slices {

constexpr int NT = 64;                 // tokens per chunk
constexpr int64_t kSeqCost = 288;      // positions charged per sequence

MLA_HD int64_t lmin(int64_t a, int64_t b) { return a < b ? a : b; }
MLA_HD int64_t lmax(int64_t a, int64_t b) { return a > b ? a : b; }

// Tokens of the stream (clamped to what B sequences of at most max_ctx hold).
MLA_HD int64_t stream_tokens(const int32_t* cu, int B, int max_ctx) {
  return lmin(lmax((int64_t)cu[B] - cu[0], 0), (int64_t)B * max_ctx);
}

MLA_HD int64_t slice_len(int64_t charged, int n_units, int min_len) {
  return lmax((charged + n_units - 1) / n_units, (int64_t)min_len);
}

struct Slice {
  int64_t r0, r1, L;   // positions [r0, r1) of the charged stream
};

MLA_HD Slice unit_slice(const int32_t* cu, int B, int max_ctx, int u, int n_units, int min_len) {
  const int64_t T = stream_tokens(cu, B, max_ctx) + (int64_t)B * kSeqCost;
  Slice s;
  s.L = slice_len(T, n_units, min_len);
  s.r0 = lmin((int64_t)u * s.L, T);
  s.r1 = lmin(s.r0 + s.L, T);
  return s;
}

// First sequence whose positions reach past position r (cu_ctx is
// non-decreasing for valid input; any input gives an index in [0, B)).
MLA_HD int seq_at(const int32_t* cu, int B, int64_t r) {
  int lo = 0, hi = B - 1;
  const int64_t c0 = cu[0];
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)cu[mid + 1] - c0 + (int64_t)(mid + 1) * kSeqCost <= r) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

struct Seg {
  int b, n, t0, tcount, nch, slot;
  int64_t start;       // cache row of the sequence's token 0
  bool whole;          // the segment covers the whole sequence
};

// Segment of sequence b in the slice of unit u; nch = 0 when it is empty or
// the sequence is invalid (the combine kernel reports those).
MLA_HD Seg seg_info(const int32_t* cu, int b, int max_ctx, const Slice& sl, int u) {
  Seg s;
  s.b = b;
  const int64_t c0 = cu[0], cb = (int64_t)cu[b] - c0, ce = (int64_t)cu[b + 1] - c0;
  s.start = cu[b];
  const int64_t n = ce - cb;
  const int64_t vs = cb + (int64_t)b * kSeqCost, v0 = vs + kSeqCost;   // charge, tokens
  const int64_t s0 = lmax(sl.r0, v0), s1 = lmin(sl.r1, v0 + n);
  s.n = (int)lmin(lmax(n, 0), (int64_t)max_ctx);
  s.t0 = (int)lmax(s0 - v0, 0);
  s.tcount = (int)lmax(s1 - s0, 0);
  if (n < 1 || n > max_ctx) s.tcount = 0;
  s.nch = (s.tcount + NT - 1) / NT;
  s.whole = s.t0 == 0 && s.tcount == n;
  s.slot = 2 * u + (vs > sl.r0 ? 1 : 0);
  return s;
}

// Walks the non-empty segments of a unit in order.
struct SegCursor {
  int k, kk;           // sequence offset from b0, ordinal among non-empty segments
  int j;               // chunk within the segment
  Seg s;
  bool done;
  MLA_HD void seek(const int32_t* cu, int b0, int b1, int max_ctx, const Slice& sl, int u) {
    for (; b0 + k < b1; ++k) {
      s = seg_info(cu, b0 + k, max_ctx, sl, u);
      if (s.nch > 0) { done = false; return; }
    }
    done = true;
  }
  MLA_HD void start(const int32_t* cu, int b0, int b1, int max_ctx, const Slice& sl, int u) {
    k = 0; kk = 0; j = 0;
    seek(cu, b0, b1, max_ctx, sl, u);
  }
  MLA_HD void next_seg(const int32_t* cu, int b0, int b1, int max_ctx, const Slice& sl, int u) {
    j = 0; ++k; ++kk;
    seek(cu, b0, b1, max_ctx, sl, u);
  }
  // next chunk; true when it starts a new segment
  MLA_HD bool next(const int32_t* cu, int b0, int b1, int max_ctx, const Slice& sl, int u) {
    if (++j < s.nch) return false;
    j = 0; ++k; ++kk;
    seek(cu, b0, b1, max_ctx, sl, u);
    return true;
  }
};

// The units whose slices hold tokens of sequence b (the combine kernel's
// view): u0 .. u1, unit u's partial in slot 2u + (vs_b > u L).  valid is
// false for a sequence outside [1, max_ctx] tokens or outside the stream.
struct SeqUnits {
  bool valid;
  int u0, u1;
  int64_t vs, L;
};

MLA_HD SeqUnits seq_units(const int32_t* cu, int b, int B, int max_ctx, int n_units,
                          int min_len) {
  SeqUnits r;
  const int64_t c0 = cu[0], cb = (int64_t)cu[b] - c0, ce = (int64_t)cu[b + 1] - c0;
  const int64_t Tt = stream_tokens(cu, B, max_ctx);
  r.valid = !(ce - cb < 1 || ce - cb > max_ctx || cb < 0 || ce > Tt);
  r.L = slice_len(Tt + (int64_t)B * kSeqCost, n_units, min_len);
  r.vs = cb + (int64_t)b * kSeqCost;
  const int64_t v0 = r.vs + kSeqCost;
  r.u0 = (int)(v0 / r.L);
  r.u1 = (int)((v0 + (ce - cb) - 1) / r.L);
  return r;
}

MLA_HD int seq_slot(const SeqUnits& r, int u) {
  return 2 * u + (r.vs > (int64_t)u * r.L ? 1 : 0);
}

}  // namespace slices
}  // namespace mla
