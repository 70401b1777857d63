// pa_span.h -- the visible-span rule, shared by the host dispatcher and the
// kernels (host and device).
#pragma once

#ifdef __CUDACC__
#define PA_HD __host__ __device__ __forceinline__
#else
#define PA_HD inline
#endif

namespace pa {

// ---------------------------------------------------------------------------
// Visible span of a query token.
//
// gllm PR #116 "feat(backend): sliding-window PagedAttention", section "What
// changes": with window > 0 the token at position p attends to positions
// p-window+1 .. p; window 0 keeps unlimited causal attention; the visible
// range starts at max(0, end-window).  A row with seqLen S and queryLen L
// holds its L new tokens at positions S-L .. S-1 (they are part of S), so
// token i sits at p = S-L+i and sees [lo, p+1).
// ---------------------------------------------------------------------------
PA_HD void query_range(int S, int L, int i, int w,
                                                     int& lo, int& hi) {
  const int end = S - L + i + 1;
  hi = end;
  lo = (w > 0) ? (end - w > 0 ? end - w : 0) : 0;
}

// First position any query token of the row sees (token 0 has the lowest lo).
PA_HD int union_lo(int S, int L, int w) {
  int lo, hi;
  query_range(S, L, 0, w, lo, hi);
  return lo;
}

// Number of positions the row's query tokens see together: [union_lo, S).
PA_HD int union_span(int S, int L, int w) {
  return S - union_lo(S, L, w);
}

}  // namespace pa
