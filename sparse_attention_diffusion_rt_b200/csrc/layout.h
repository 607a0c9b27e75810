// Host-side checks of the strided [B, H, L, d] layout shared by Q, K, V, O
// and R: that no two (b, h, l) rows share an element (so that the CTAs that
// store different rows never race), and the byte span a tensor covers (so
// that an output that overlaps an input or another output is refused).
#pragma once
#include <algorithm>
#include <cstdint>

#include "rt.h"

namespace rtb {

// True when the rows of the layout are pairwise disjoint.  The dimensions of
// extent > 1, with the row itself (d elements, stride 1) innermost, are sorted
// by stride; each stride must then reach past everything the smaller strides
// span.  This accepts every permuted dense layout ([B,H,L,d], [B,L,H,d], head
// slices of either) and rejects layouts whose heads or batches alias.
inline bool layout_rows_disjoint(const rt_attn_desc& d) {
  struct Dim {
    long long extent, stride;
  };
  Dim dims[4] = {{d.d, 1}, {d.L, d.stride_l}, {d.H, d.stride_h}, {d.B, d.stride_b}};
  int n = 1;
  for (int i = 1; i < 4; ++i)
    if (dims[i].extent > 1) dims[n++] = dims[i];
  std::sort(dims, dims + n, [](const Dim& a, const Dim& b) { return a.stride < b.stride; });
  long long reach = dims[0].extent * dims[0].stride;     // elements spanned by the inner dimensions
  for (int i = 1; i < n; ++i) {
    if (dims[i].stride < reach) return false;
    reach = dims[i].stride * (dims[i].extent - 1) + reach;
  }
  return true;
}

// Bytes from the first to one past the last element a tensor of this layout covers.
inline long long layout_span_bytes(const rt_attn_desc& d, int elem_bytes) {
  const long long last = (static_cast<long long>(d.B) - 1) * d.stride_b + (static_cast<long long>(d.H) - 1) * d.stride_h +
                         (static_cast<long long>(d.L) - 1) * d.stride_l + d.d;
  return last * elem_bytes;
}

// Whether [a, a + na) and [b, b + nb) share a byte (a NULL range shares none).
inline bool ranges_overlap(const void* a, long long na, const void* b, long long nb) {
  if (!a || !b) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + static_cast<uintptr_t>(nb) && y < x + static_cast<uintptr_t>(na);
}

}  // namespace rtb
