// Tensor maps the fine block-sparse kernels load their tiles through.
#pragma once

#include <cuda.h>

namespace vsa {

// All over the tiled [B*H*64C rows, d] bf16 tensors, 128-byte swizzle,
// 64-column boxes: q, k, v with 64-row boxes (one cube), k16, v16 with
// 16-row boxes (the valid rows of a cube with at most 16 tokens).
struct FineMaps {
  CUtensorMap q, k, v, k16, v16;
};

// The fine backward's maps, 64-row boxes: tiled q, k, v and the tiled
// gradient of the fine output (dO_f).
struct BwdMaps {
  CUtensorMap q, k, v, dO;
};

}  // namespace vsa
