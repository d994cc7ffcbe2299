// Workspace layout of the linear compensation branch (csrc/linear.cu).
#pragma once

#include <cstddef>

namespace vsa {

// Byte offsets inside the caller's workspace: phi(q) and phi(k) (bf16,
// [B H, N, d]), the per-chunk [KV | z] partials (float32, [B H][splits][128]
// [d + 16]), the bf16 matrix B = [KV^T ; z^T ; 0] ([B H][d + 16][d]); splits
// chunks of `per` tokens per sequence.
struct LinearLayout {
  int splits, per;
  size_t fq, fk, partial, bmat, bytes;
};

LinearLayout linear_layout(int bh, long long N, int d);

}  // namespace vsa
