// tail.cuh -- kernels of the group-shared fixed fan-in sparse tail (HASTE,
// "Hardware-Aware Dynamic Sparse Training for Large Output Spaces", Methodology 1:
// labels in groups of G share one fan-in index set I_g of k features; every label
// keeps its own weight row).  The gather-once / dense-MMA pattern of the page's
// "hardware alignment" paragraph maps onto sm_100a as: the k feature rows of the
// feature-major input X^T [d, Bp] named by I_g are gathered once per group into a
// 128B-swizzled shared-memory tile, and every MMA of the group (forward, dW, dX)
// reads that tile through tcgen05 descriptors with fp32 accumulation in TMEM.
//
// Shared-memory tile layouts (E = element bytes, R = 128/E elements per 128B row):
//   Xg  : gathered X^T rows.  Byte offset of (slot s, batch b) before swizzle:
//         (b / R) * SR * 128 + s * 128 + (b % R) * E, SR = rows per b-block.
//         Read as an MN-major A operand (forward, M = batch) and as a K-major A
//         operand (dW, M = slot) -- the same bytes serve both.
//   Wg  : W rows of the group.  (label j, slot s): (s / R) * G * 128 + j * 128 +
//         (s % R) * E, swizzled.  K-major B of the forward (N = label) and
//         MN-major B of the dX product (N = slot).
//   dY  : no-swizzle 8x16B core matrices.  (batch b, label j): (j / CW) * BT * 16 +
//         b * 16 + (j % CW) * E with CW = 16/E, BT = batch rows of the tile.
//         MN-major B of dW (N = label, K = batch), K-major A of the dX product
//         (M = batch, K = label).
#pragma once

#include "common.cuh"

namespace haste {

struct TailShape {
  int B, Bp, d, G, k;
  int64_t n_groups, L;
};

// Per-launch arguments of the tail kernels.
struct TailArgs {
  TailShape sh;
  const int32_t* idx;      // [n_groups, k] device
  const void* Xt;          // [d, Bp] feature-major input, zero padded
  const void* W;           // [L, k]
  const void* dY;          // [B, L]   (given-gradient calls, or fused-step buffer)
  void* logits;            // [B, L]   forward output
  void* dW;                // [L, k]
  void* dY_out;            // [B, L]   fused step: gradient written for the dX pass
  float* dX_part;          // [n_chunks, d, Bp] partial sums of the dX pass
  float* loss_part;        // [gridDim.x] per-CTA loss partials (fused step)
  const int32_t* pos_ptr;  // [B+1] tail positives CSR (fused step)
  const int32_t* pos_ids;  // [nnz]
  float grad_scale;
  int band;                // dX: features per band
  int n_bands;
  int n_chunks;
};

}  // namespace haste
