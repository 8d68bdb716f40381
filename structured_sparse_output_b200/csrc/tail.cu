// tail.cu -- sm_100a kernels of the group-shared fixed fan-in sparse tail.
//
// HASTE ("Hardware-Aware Dynamic Sparse Training for Large Output Spaces"),
// Methodology 1: labels are split into groups of G; all labels of group g share
// one sorted fan-in set I_g of k features and keep their own weight row.
//   forward : logits_g = X[:, I_g] . W_g^T
//   dW      : dW_g     = dY_g^T . X[:, I_g]
//   dX      : dX[:, I_g] += dY_g . W_g
// The page's "gather-once and dense MMA" pattern: X[:, I_g] is staged into shared
// memory once per group and every product of the group runs on the tensor cores.
// The shared-memory layouts are described in tail.cuh.
#include "tail.cuh"

namespace haste {

namespace {

constexpr int kThreads = 128;  // 4 warps = the 128 TMEM lanes of the epilogue

__host__ __device__ constexpr uint32_t tmem_cols_for(uint32_t n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

// ----------------------------------------------------------------- loaders
// Gather rows idx_s[0..nrows) of X^T (row length Bp) for batch columns
// [b0, b0 + nb) into the swizzled Xg layout (SR rows per b-block).
template <typename T, bool kMN>
__device__ __forceinline__ void gather_xg(uint32_t xg, const T* __restrict__ Xt, const int32_t* idx_s,
                                          int nrows, int Bp, int b0, int nb, int SR) {
  constexpr int R = 128 / sizeof(T), CW = 16 / sizeof(T);
  const int total = (nb / R) * nrows * 8;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int c = i & 7, rs = i >> 3;
    const int s = rs % nrows, bb = rs / nrows;
    const T* src = Xt + (int64_t)idx_s[s] * Bp + b0 + bb * R + c * CW;
    cp_async16(xg + swz<T, kMN>((uint32_t)(bb * SR * 128 + s * 128 + c * 16)), src, 16);
  }
}

// The G x k weight block of group g (contiguous in W) into the swizzled Wg layout.
template <typename T, bool kMN>
__device__ __forceinline__ void load_wg(uint32_t wg, const T* __restrict__ W, int64_t g, int G, int k) {
  constexpr int CW = 16 / sizeof(T);
  const int cpr = k / CW;  // 16-byte chunks per weight row
  const T* src0 = W + g * (int64_t)G * k;
  for (int i = threadIdx.x; i < G * cpr; i += blockDim.x) {
    const int j = i / cpr, cc = i % cpr;
    const uint32_t off = (uint32_t)((cc >> 3) * G * 128 + j * 128 + (cc & 7) * 16);
    cp_async16(wg + swz<T, kMN>(off), src0 + (int64_t)j * k + cc * CW, 16);
  }
}

// dY[b0 + b, col0 + j] for b < BT (zero for rows at or beyond B), j < G, into the
// no-swizzle core layout (K-major A operand of the dX product; for bf16 also the
// MN-major B operand of dW).  Lane pairs fetch one 32-byte sector.
template <typename T>
__device__ __forceinline__ void load_dy_k(uint32_t dy, const T* __restrict__ dY, int64_t L, int B, int b0, int BT,
                                          int64_t col0, int G) {
  constexpr int CW = 16 / sizeof(T);
  const int nch = G / CW;
  for (int i = threadIdx.x; i < BT * nch; i += blockDim.x) {
    const int rest = i >> 1;
    const int b = rest % BT, jc = (rest / BT) * 2 + (i & 1);
    const bool in = (b0 + b) < B;
    const T* src = in ? dY + (int64_t)(b0 + b) * L + col0 + jc * CW : dY;
    cp_async16(dy + (uint32_t)(jc * BT * 16 + b * 16), src, in ? 16u : 0u);
  }
}

// Shared-memory bytes of the dY tile read as the MN-major B operand of dW.
template <typename T>
__host__ __device__ constexpr uint32_t dy_mn_bytes(int BT, int G) {
  return sizeof(T) == 4 ? (uint32_t)((G + 31) / 32) * BT * 128 : (uint32_t)BT * G * sizeof(T);
}
// Offset of element (b, j) of that tile: bf16 keeps the no-swizzle core layout;
// fp32 (tf32) uses 128-byte rows of 32 labels per batch row, 32B-granular swizzle.
template <typename T>
__device__ __forceinline__ uint32_t dy_mn_off(int b, int j, int BT) {
  if constexpr (sizeof(T) == 4) return sw128_32b((uint32_t)((j >> 5) * BT * 128 + b * 128 + (j & 31) * 4));
  else return (uint32_t)((j / 8) * BT * 16 + b * 16 + (j % 8) * 2);
}

template <typename T>
__device__ __forceinline__ void load_dy_mn(uint32_t dy, const T* __restrict__ dY, int64_t L, int B, int b0, int BT,
                                           int64_t col0, int G) {
  if constexpr (sizeof(T) == 2) {
    load_dy_k<T>(dy, dY, L, B, b0, BT, col0, G);
  } else {
    constexpr int CW = 4;
    const int nch = G / CW;
    for (int i = threadIdx.x; i < BT * nch; i += blockDim.x) {
      const int b = i / nch, jc = i % nch;
      const bool in = (b0 + b) < B;
      const T* src = in ? dY + (int64_t)(b0 + b) * L + col0 + jc * CW : dY;
      cp_async16(dy + dy_mn_off<T>(b, jc * CW, BT), src, in ? 16u : 0u);
    }
  }
}

// Finish the cp.async copies of this thread and publish them to the tensor core.
__device__ __forceinline__ void staged_smem_ready() {
  cp_async_commit();
  cp_async_wait_all();
  fence_proxy_async_smem();
  __syncthreads();
}

// ------------------------------------------------------------ MMA issue
// Forward: D[128 batch x G] = Xg(b-tile, MN-major) x Wg^T (K-major).
template <typename T>
__device__ __forceinline__ void issue_forward(uint32_t d_tmem, uint32_t xg_tile, uint32_t wg, int SR, int G,
                                              int k) {
  constexpr int R = 128 / sizeof(T), KI = Elem<T>::kMmaK;
  const uint32_t idesc = make_idesc(Elem<T>::kFmt, 1, 0, 128, (uint32_t)G);
  for (int kk = 0; kk < k / KI; ++kk) {
    const uint64_t a = mn_desc<T>(xg_tile + kk * KI * 128, (uint32_t)SR * 128);
    const uint32_t boff = (uint32_t)(((kk * KI) / R) * G * 128 + (kk % (R / KI)) * 32);
    const uint64_t b = make_sdesc(wg + boff, 16, 1024, kLayoutSw128);
    mma_ss<Elem<T>::kTF32>(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// N of the dW product: G, rounded up to whole 32-label atoms for tf32 (whose
// MN-major operand layout is 32 elements wide); extra columns are ignored.
template <typename T>
__host__ __device__ constexpr int dw_n(int G) {
  return sizeof(T) == 4 ? (G + 31) / 32 * 32 : G;
}

// dW: D[128 slots x G] = Xg^T (K-major, M = slot) x dY (MN-major, N = label), K = BT.
template <typename T>
__device__ __forceinline__ void issue_dw(uint32_t d_tmem, uint32_t xg, uint32_t dy, int SR, int BT, int G) {
  constexpr int R = 128 / sizeof(T), KI = Elem<T>::kMmaK;
  const uint32_t idesc = make_idesc(Elem<T>::kFmt, 0, 1, 128, (uint32_t)dw_n<T>(G));
  for (int kk = 0; kk < BT / KI; ++kk) {
    const int b = kk * KI;
    const uint64_t a =
        make_sdesc(xg + (uint32_t)((b / R) * SR * 128 + (kk % (R / KI)) * 32), 16, 1024, kLayoutSw128);
    uint64_t bd;
    if constexpr (sizeof(T) == 4) bd = mn_desc<T>(dy + (uint32_t)(b * 128), (uint32_t)BT * 128);
    else bd = make_sdesc(dy + (uint32_t)((b / 8) * 128), 128, (uint32_t)BT * 16, kLayoutNone);
    mma_ss<Elem<T>::kTF32>(d_tmem, a, bd, idesc, kk > 0 ? 1u : 0u);
  }
}

// dX product: Z[128 batch x N slots] = dY (K-major A, M = batch, K = label) x
// Wg[:, s0 : s0+N] (MN-major B, N = slot).  s0 is a multiple of the 128B row.
template <typename T>
__device__ __forceinline__ void issue_z(uint32_t d_tmem, uint32_t dy, uint32_t wg, int BT, int G, int s0, int N) {
  constexpr int R = 128 / sizeof(T), KI = Elem<T>::kMmaK, CW = 16 / sizeof(T);
  const uint32_t idesc = make_idesc(Elem<T>::kFmt, 0, 1, 128, (uint32_t)N);
  for (int kk = 0; kk < G / KI; ++kk) {
    const int j = kk * KI;
    const uint64_t a = make_sdesc(dy + (uint32_t)((j / CW) * BT * 16), (uint32_t)BT * 16, 128, kLayoutNone);
    const uint64_t b = mn_desc<T>(wg + (uint32_t)((s0 / R) * G * 128 + j * 128), (uint32_t)G * 128);
    mma_ss<Elem<T>::kTF32>(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// Bounded wait of the whole block on an MMA-completion barrier; returns false on
// timeout (every thread sees the same outcome).
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t& phase, int* abort_flag) {
  const bool ok = mbar_wait(bar, phase);
  phase ^= 1u;
  if (!ok) *abort_flag = 1;
  tc_fence_after();
  __syncthreads();
  return *abort_flag == 0;
}

__device__ __forceinline__ void load_idx_row(int32_t* idx_s, const int32_t* __restrict__ idx, int64_t g, int k) {
  for (int s = threadIdx.x; s < k; s += blockDim.x) idx_s[s] = idx[g * k + s];
}

// TMEM allocation by warp 0; the address is published through shared memory.
__device__ __forceinline__ uint32_t tmem_setup(uint32_t* slot, uint32_t ncols) {
  if (threadIdx.x < 32) {
    tmem_alloc(slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *slot;
}

__device__ __forceinline__ void tmem_teardown(uint32_t taddr, uint32_t ncols) {
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(taddr, ncols);
  }
}

__device__ __forceinline__ uint32_t lane_base(uint32_t tmem) { return tmem + (((threadIdx.x / 32) * 32u) << 16); }

}  // namespace

// =========================================================================
// X [B, d] -> X^T [d, Bp] (zero for b >= B): makes each gathered feature a
// contiguous row of Bp elements.
template <typename T>
__global__ void __launch_bounds__(256) k_xt(const T* __restrict__ X, T* __restrict__ Xt, int B, int Bp, int d) {
  __shared__ T tile[32][33];
  const int f0 = blockIdx.x * 32, b0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int b = b0 + i, f = f0 + tx;
    tile[i][tx] = (b < B && f < d) ? X[(int64_t)b * d + f] : Elem<T>::from_f(0.f);
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int f = f0 + i, b = b0 + tx;
    if (f < d && b < Bp) Xt[(int64_t)f * Bp + b] = tile[tx][i];
  }
}

// =========================================================================
// Forward with materialised logits.  Work item = (group, 128-row batch tile).
template <typename T>
__global__ void __launch_bounds__(kThreads, 1) k_forward(TailArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TailShape sh = a.sh;
  const int G = sh.G, k = sh.k, SR = k;
  constexpr int R = 128 / sizeof(T);
  const uint32_t base = align1024(smem_u32(smem));
  const uint32_t xg = base;
  const uint32_t wg = xg + (128 / R) * SR * 128;
  uint8_t* gen = smem + (wg + (uint32_t)G * k * sizeof(T) - smem_u32(smem));
  int32_t* idx_s = reinterpret_cast<int32_t*>(gen);
  uint64_t* bar = reinterpret_cast<uint64_t*>(gen + ((k * 4 + 7) & ~7));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t ncols = tmem_cols_for(G);
  const uint32_t tmem = tmem_setup(tslot, ncols);
  uint32_t phase = 0;
  const int n_bt = sh.Bp / 128;
  const int64_t items = sh.n_groups * n_bt;
  const T* Xt = static_cast<const T*>(a.Xt);
  const T* W = static_cast<const T*>(a.W);
  T* out = static_cast<T*>(a.logits);

  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t g = it / n_bt;
    const int t = (int)(it % n_bt);
    load_idx_row(idx_s, a.idx, g, k);
    __syncthreads();
    gather_xg<T, true>(xg, Xt, idx_s, k, sh.Bp, t * 128, 128, SR);
    load_wg<T, false>(wg, W, g, G, k);
    staged_smem_ready();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_forward<T>(tmem, xg, wg, SR, G, k);
      mma_commit(bar);
    }
    if (!block_wait(bar, phase, abort_flag)) break;
    // epilogue: thread = batch row of the tile, columns = labels of the group
    const int b = t * 128 + threadIdx.x;
    for (int c = 0; c < G; c += 16) {
      float v[16];
      tmem_ld16(lane_base(tmem) + c, v);
      tmem_wait_ld();
      if (b < sh.B) {
        T* dst = out + (int64_t)b * sh.L + g * G + c;
        if constexpr (sizeof(T) == 2) {
          uint4 p0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                pack_bf16x2(v[6], v[7]));
          uint4 p1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                pack_bf16x2(v[14], v[15]));
          reinterpret_cast<uint4*>(dst)[0] = p0;
          reinterpret_cast<uint4*>(dst)[1] = p1;
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  tmem_teardown(tmem, ncols);
}

// =========================================================================
// dW with a given upstream gradient.  Work item = group; K of the product is the
// whole (padded) batch.
template <typename T>
__global__ void __launch_bounds__(kThreads, 1) k_backward_dw(TailArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TailShape sh = a.sh;
  const int G = sh.G, k = sh.k, SR = k, Bp = sh.Bp;
  constexpr int R = 128 / sizeof(T);
  const uint32_t base = align1024(smem_u32(smem));
  const uint32_t xg = base;
  const uint32_t xg_bytes = (uint32_t)((Bp / R) * SR * 128 + (k < 128 ? (128 - k) * 128 : 0));
  const uint32_t dy = xg + xg_bytes;
  uint8_t* gen = smem + (dy + dy_mn_bytes<T>(Bp, G) - smem_u32(smem));
  int32_t* idx_s = reinterpret_cast<int32_t*>(gen);
  uint64_t* bar = reinterpret_cast<uint64_t*>(gen + ((k * 4 + 7) & ~7));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t ncols = tmem_cols_for((uint32_t)dw_n<T>(G));
  const uint32_t tmem = tmem_setup(tslot, ncols);
  uint32_t phase = 0;
  const T* Xt = static_cast<const T*>(a.Xt);
  const T* dYp = static_cast<const T*>(a.dY);
  T* dW = static_cast<T*>(a.dW);

  for (int64_t g = blockIdx.x; g < sh.n_groups; g += gridDim.x) {
    load_idx_row(idx_s, a.idx, g, k);
    __syncthreads();
    gather_xg<T, false>(xg, Xt, idx_s, k, Bp, 0, Bp, SR);
    load_dy_mn<T>(dy, dYp, sh.L, sh.B, 0, Bp, g * G, G);
    staged_smem_ready();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_dw<T>(tmem, xg, dy, SR, Bp, G);
      mma_commit(bar);
    }
    if (!block_wait(bar, phase, abort_flag)) break;
    // epilogue: thread = slot s, columns = labels j; dW[g*G+j, s]
    const int s = threadIdx.x;
    for (int c = 0; c < G; c += 16) {
      float v[16];
      tmem_ld16(lane_base(tmem) + c, v);
      tmem_wait_ld();
      if (s < k) {
        T* dst = dW + (g * G + c) * (int64_t)k + s;
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[(int64_t)i * k] = Elem<T>::from_f(v[i]);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  tmem_teardown(tmem, ncols);
}

// =========================================================================
// dX pass.  CTA = (128-row batch tile t, feature band h, group chunk c).  For each
// group of the chunk: Z = dY_g(tile) . W_g[:, slots of the band] on the tensor
// cores, then thread b adds row b of Z into its own column of the band's fp32
// accumulator in shared memory, slot s going to feature idx[g, s].  A thread owns
// its batch column outright, so every feature receives its (group, slot) terms in
// ascending group order -- the order of the feature's inverse-map segment -- with
// no atomics.  The chunk's accumulator is written to dX_part[c]; k_dx_reduce sums
// the chunks in ascending order.
template <typename T, bool kFromStepBuffer>
__global__ void __launch_bounds__(kThreads, 1) k_backward_dx(TailArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TailShape sh = a.sh;
  const int G = sh.G, k = sh.k;
  constexpr int R = 128 / sizeof(T);
  const int n_bt = sh.Bp / 128;
  const int per_chunk = n_bt * a.n_bands;
  const int c = blockIdx.x / per_chunk;
  const int h = (blockIdx.x % per_chunk) / n_bt;
  const int t = blockIdx.x % n_bt;
  const int f0 = h * a.band;
  const int f1 = min(sh.d, f0 + a.band);
  const int64_t g0 = (int64_t)c * sh.n_groups / a.n_chunks;
  const int64_t g1 = (int64_t)(c + 1) * sh.n_groups / a.n_chunks;

  const uint32_t base = align1024(smem_u32(smem));
  const uint32_t wg = base;
  const uint32_t dy = wg + (uint32_t)G * k * sizeof(T);
  uint8_t* gen = smem + (dy + 128u * G * sizeof(T) - smem_u32(smem));
  float* acc = reinterpret_cast<float*>(gen);
  int32_t* idx_s = reinterpret_cast<int32_t*>(acc + (size_t)a.band * 128);
  uint64_t* bar = reinterpret_cast<uint64_t*>(idx_s + ((k + 1) & ~1));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  int* range_s = abort_flag + 1;  // [s_lo, s_hi]

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < a.band * 128; i += blockDim.x) acc[i] = 0.f;
  const uint32_t ncols = tmem_cols_for((uint32_t)k);
  const uint32_t tmem = tmem_setup(tslot, ncols);
  uint32_t phase = 0;
  const T* W = static_cast<const T*>(a.W);
  const T* dYp = static_cast<const T*>(kFromStepBuffer ? a.dY_out : a.dY);
  const int b = threadIdx.x;

  for (int64_t g = g0; g < g1; ++g) {
    load_idx_row(idx_s, a.idx, g, k);
    __syncthreads();
    if (threadIdx.x < 32) {
      // slot range of the band: idx is sorted, so it is [#(idx < f0), #(idx < f1))
      int lo = 0, hi = 0;
      for (int s = threadIdx.x; s < k; s += 32) {
        lo += __popc(__ballot_sync(0xffffffffu, idx_s[s] < f0));
        hi += __popc(__ballot_sync(0xffffffffu, idx_s[s] < f1));
      }
      if (threadIdx.x == 0) {
        range_s[0] = lo;
        range_s[1] = hi;
      }
    }
    __syncthreads();
    const int s_lo = range_s[0], s_hi = range_s[1];
    if (s_hi == s_lo) continue;  // uniform: no feature of this band in the group
    const int s0 = s_lo & ~(R - 1);
    const int N = ((s_hi - s0 + R - 1) / R) * R;
    load_wg<T, true>(wg, W, g, G, k);
    load_dy_k<T>(dy, dYp, sh.L, sh.B, t * 128, 128, g * G, G);
    staged_smem_ready();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_z<T>(tmem, dy, wg, 128, G, s0, N);
      mma_commit(bar);
    }
    if (!block_wait(bar, phase, abort_flag)) break;
    for (int cc = (s_lo - s0) & ~15; cc < s_hi - s0; cc += 16) {
      float v[16];
      tmem_ld16(lane_base(tmem) + cc, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int s = s0 + cc + i;
        if (s >= s_lo && s < s_hi) acc[(idx_s[s] - f0) * 128 + b] += v[i];
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  __syncthreads();
  // chunk partial: dX_part[c, f, t*128 + b]
  for (int f = f0; f < f1; ++f)
    a.dX_part[((int64_t)c * sh.d + f) * sh.Bp + t * 128 + b] = acc[(f - f0) * 128 + b];
  tmem_teardown(tmem, ncols);
}

// One warp: *loss = scale * sum of part[0..n) in fp64, in a fixed order (lane j
// adds part[j], part[j+32], ... in turn, then a butterfly over the lanes), so
// the result is the same on every run.
__device__ __forceinline__ void loss_sum(const float* __restrict__ part, int n, float scale, float* loss) {
  double t = 0.0;
  for (int i = (int)(threadIdx.x & 31); i < n; i += 32) t += (double)part[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  if ((threadIdx.x & 31) == 0) *loss = (float)(t * (double)scale);
}

// dX[b, f] (+)= sum over chunks c ascending of dX_part[c, f, b].  With
// loss_part, the first warp of block (0, 0) also writes the loss, as
// k_loss_reduce does.
__global__ void __launch_bounds__(256) k_dx_reduce(const float* __restrict__ P, float* __restrict__ dX, int C,
                                                   int d, int Bp, int B, int accumulate,
                                                   const float* __restrict__ loss_part, int n_loss, float scale,
                                                   float* __restrict__ loss) {
  // block: 8 feature rows x 128 batch columns; warp w sums feature f0 + w, lane l
  // the 4 batch columns 4l.. as one 16-byte load per chunk (eight loads in flight);
  // every element adds its chunks in ascending order
  __shared__ float tile[8][128 + 4];
  const int f0 = blockIdx.x * 8, b0 = blockIdx.y * 128;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (loss_part && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 32) loss_sum(loss_part, n_loss, scale, loss);
  const int64_t cs = (int64_t)d * Bp;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (f0 + w < d) {
    const float4* p = reinterpret_cast<const float4*>(P + (int64_t)(f0 + w) * Bp + b0) + l;
#pragma unroll 8
    for (int c = 0; c < C; ++c) {
      const float4 v = p[c * (cs / 4)];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
  }
  tile[w][4 * l] = acc.x;
  tile[w][4 * l + 1] = acc.y;
  tile[w][4 * l + 2] = acc.z;
  tile[w][4 * l + 3] = acc.w;
  __syncthreads();
  // dX rows: eight consecutive features of one batch row per group of 8 threads
  for (int i = threadIdx.x; i < 8 * 128; i += 256) {
    const int bb = b0 + i / 8, f = f0 + (i & 7);
    if (bb < B && f < d) {
      const float v = tile[i & 7][i / 8];
      float* q = dX + (int64_t)bb * d + f;
      *q = accumulate ? *q + v : v;
    }
  }
}

// =========================================================================
// Fused tail step, pass 1.  Work item = group, whole batch:
//   gather X[:, I_g] once -> forward MMA per 128-row tile -> BCE epilogue in
//   registers (logits never leave TMEM) -> dY_g to shared memory (and to the
//   dY buffer read by the dX pass) -> dW MMA from the same gathered tile.
// BCE with logits against sparse positives: dY = scale * (sigmoid(z) - y),
// loss = scale * sum(softplus(z) - z*y).  sigmoid comes from one tanh
// (sigmoid(z) = 0.5 + 0.5 tanh(z/2)); the softplus sum of a row segment is
// sum(max(z,0)) - log(prod sigmoid(|z|)), one log per 32 labels.
template <typename T>
__global__ void __launch_bounds__(kThreads, 1) k_step(TailArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TailShape sh = a.sh;
  const int G = sh.G, k = sh.k, SR = k, Bp = sh.Bp;
  constexpr int R = 128 / sizeof(T), CW = 16 / sizeof(T);
  const int n_bt = Bp / 128;
  const uint32_t base = align1024(smem_u32(smem));
  const uint32_t xg = base;
  const uint32_t xg_bytes = (uint32_t)((Bp / R) * SR * 128 + (k < 128 ? (128 - k) * 128 : 0));
  // fp32: the tf32 forward needs the gathered tile in the 32B-granular MN-major
  // swizzle, which the K-major dW view cannot read, so it is gathered twice.
  const uint32_t xg_mn = sizeof(T) == 4 ? xg + xg_bytes : xg;
  const uint32_t wg = xg + (sizeof(T) == 4 ? 2 : 1) * xg_bytes;
  const uint32_t dy = wg + (uint32_t)G * k * sizeof(T);
  uint8_t* gen = smem + (dy + dy_mn_bytes<T>(Bp, G) - smem_u32(smem));
  int32_t* idx_s = reinterpret_cast<int32_t*>(gen);
  uint64_t* bar = reinterpret_cast<uint64_t*>(gen + ((k * 4 + 7) & ~7));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  float* red = reinterpret_cast<float*>(abort_flag + 1);  // 4 warp partials

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t ncols = tmem_cols_for((uint32_t)(n_bt * G + dw_n<T>(G)));
  const uint32_t tmem = tmem_setup(tslot, ncols);
  const uint32_t tmem_dw = tmem + (uint32_t)(n_bt * G);
  uint32_t phase = 0;
  const T* Xt = static_cast<const T*>(a.Xt);
  const T* W = static_cast<const T*>(a.W);
  T* dY_out = static_cast<T*>(a.dY_out);
  T* dW = static_cast<T*>(a.dW);
  const float scale = a.grad_scale;
  float loss_acc = 0.f;

  for (int64_t g = blockIdx.x; g < sh.n_groups; g += gridDim.x) {
    load_idx_row(idx_s, a.idx, g, k);
    __syncthreads();
    gather_xg<T, false>(xg, Xt, idx_s, k, Bp, 0, Bp, SR);
    if constexpr (sizeof(T) == 4) gather_xg<T, true>(xg_mn, Xt, idx_s, k, Bp, 0, Bp, SR);
    load_wg<T, false>(wg, W, g, G, k);
    staged_smem_ready();
    if (threadIdx.x == 0) {
      tc_fence_after();
      for (int t = 0; t < n_bt; ++t)
        issue_forward<T>(tmem + (uint32_t)(t * G), xg_mn + (uint32_t)(t * (128 / R) * SR * 128), wg, SR, G, k);
      mma_commit(bar);
    }
    if (!block_wait(bar, phase, abort_flag)) break;

    for (int t = 0; t < n_bt; ++t) {
      const int b = t * 128 + threadIdx.x;
      const bool live = b < sh.B;
      // positives of row b inside this group's label range -> bit mask
      uint64_t ym_lo = 0, ym_hi = 0;
      if (live) {
        const int64_t lo = g * G;
        for (int p = a.pos_ptr[b]; p < a.pos_ptr[b + 1]; ++p) {
          const int64_t l = (int64_t)a.pos_ids[p] - lo;
          if (l >= 0 && l < 64) ym_lo |= 1ull << l;
          else if (l >= 64 && l < G) ym_hi |= 1ull << (l - 64);
        }
      }
      for (int c = 0; c < G; c += 16) {
        float z[16];
        tmem_ld16(lane_base(tmem) + (uint32_t)(t * G + c), z);
        tmem_wait_ld();
        float dyv[16];
        float lin = 0.f, prod = 1.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j = c + i;
          const uint64_t m = j < 64 ? ym_lo : ym_hi;
          const float y = ((m >> (j & 63)) & 1ull) ? 1.f : 0.f;
          const float th = tanh_approx(0.5f * z[i]);
          dyv[i] = live ? scale * (fmaf(0.5f, th, 0.5f) - y) : 0.f;
          lin += fmaxf(z[i], 0.f) - z[i] * y;
          prod *= fmaf(0.5f, fabsf(th), 0.5f);
        }
        if (live) loss_acc += lin - __logf(prod);
        // dY row segment -> shared memory (dW operand layout) and the dX-pass buffer
#pragma unroll
        for (int q = 0; q < 16 / CW; ++q) {
          const uint32_t dst = dy + dy_mn_off<T>(b, c + q * CW, Bp);
          uint4 v;
          if constexpr (sizeof(T) == 2) {
            v = make_uint4(pack_bf16x2(dyv[8 * q], dyv[8 * q + 1]), pack_bf16x2(dyv[8 * q + 2], dyv[8 * q + 3]),
                           pack_bf16x2(dyv[8 * q + 4], dyv[8 * q + 5]), pack_bf16x2(dyv[8 * q + 6], dyv[8 * q + 7]));
          } else {
            v = make_uint4(__float_as_uint(dyv[4 * q]), __float_as_uint(dyv[4 * q + 1]),
                           __float_as_uint(dyv[4 * q + 2]), __float_as_uint(dyv[4 * q + 3]));
          }
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                       : "memory");
          if (live)
            *reinterpret_cast<uint4*>(dY_out + (int64_t)b * sh.L + g * G + c + q * CW) = v;
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_dw<T>(tmem_dw, xg, dy, SR, Bp, G);
      mma_commit(bar);
    }
    if (!block_wait(bar, phase, abort_flag)) break;
    const int s = threadIdx.x;
    for (int c = 0; c < G; c += 16) {
      float v[16];
      tmem_ld16(lane_base(tmem_dw) + c, v);
      tmem_wait_ld();
      if (s < k) {
        T* dst = dW + (g * G + c) * (int64_t)k + s;
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[(int64_t)i * k] = Elem<T>::from_f(v[i]);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  // deterministic block reduction of the loss: xor tree in each warp, then warps
  // in order
  float v = loss_acc;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) a.loss_part[blockIdx.x] = ((red[0] + red[1]) + red[2]) + red[3];
  tmem_teardown(tmem, ncols);
}

// loss = scale * sum of the per-CTA partials in ascending CTA order (double).
__global__ void k_loss_reduce(const float* __restrict__ part, int n, float scale, float* loss) {
  if (blockIdx.x == 0 && threadIdx.x < 32) loss_sum(part, n, scale, loss);
}

// Self-test of the bounded-wait path: one thread waits on an mbarrier that no one
// arrives on; the wait gives up after limit_ns, records kErrTimeout and returns.
__global__ void k_selftest_wait(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait(&bar, 0, limit_ns);
  }
}

// ------------------------------------------------------------- host side
namespace tail {

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t st) {
  k_selftest_wait<<<1, 32, 0, st>>>(limit_ns);
  return cudaGetLastError();
}


size_t smem_forward(int elem, int k, int G) {
  const int R = 128 / elem;
  return 1024 + (size_t)(128 / R) * k * 128 + (size_t)G * k * elem + k * 4 + 64;
}
size_t dy_mn_host(int elem, int BT, int G) { return elem == 4 ? (size_t)((G + 31) / 32) * BT * 128 : (size_t)BT * G * elem; }
size_t smem_dw(int elem, int k, int G, int Bp) {
  const int R = 128 / elem;
  return 1024 + (size_t)(Bp / R) * k * 128 + (k < 128 ? (128 - k) * 128 : 0) + dy_mn_host(elem, Bp, G) + k * 4 + 64;
}
size_t smem_dx(int elem, int k, int G, int band) {
  return 1024 + (size_t)G * k * elem + 128 * (size_t)G * elem + (size_t)band * 128 * 4 + k * 4 + 64;
}
size_t smem_step(int elem, int k, int G, int Bp) {
  const int R = 128 / elem;
  const size_t xg = (size_t)(Bp / R) * k * 128 + (k < 128 ? (128 - k) * 128 : 0);
  return 1024 + (elem == 4 ? 2 : 1) * xg + (size_t)G * k * elem + dy_mn_host(elem, Bp, G) + k * 4 + 96;
}

template <typename T>
cudaError_t launch_xt(const void* X, void* Xt, int B, int Bp, int d, cudaStream_t st) {
  dim3 grid((d + 31) / 32, Bp / 32);
  k_xt<T><<<grid, 256, 0, st>>>(static_cast<const T*>(X), static_cast<T*>(Xt), B, Bp, d);
  return cudaGetLastError();
}

template <typename Kern>
static cudaError_t launch_kernel(Kern kern, int grid, size_t smem, cudaStream_t st, const TailArgs& a) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T>
static int resident_grid(const void* kern, size_t smem, int64_t items, int sms) {
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t g = (int64_t)per_sm * sms;
  return (int)(items < g ? items : g);
}

template <typename T>
cudaError_t launch_forward(const TailArgs& a, int sms, cudaStream_t st) {
  const size_t smem = smem_forward(sizeof(T), a.sh.k, a.sh.G);
  cudaError_t e = cudaFuncSetAttribute(k_forward<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = resident_grid<T>((const void*)k_forward<T>, smem, a.sh.n_groups * (a.sh.Bp / 128), sms);
  return launch_kernel(k_forward<T>, grid, smem, st, a);
}

template <typename T>
cudaError_t launch_backward_dw(const TailArgs& a, int sms, cudaStream_t st) {
  const size_t smem = smem_dw(sizeof(T), a.sh.k, a.sh.G, a.sh.Bp);
  cudaError_t e = cudaFuncSetAttribute(k_backward_dw<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = resident_grid<T>((const void*)k_backward_dw<T>, smem, a.sh.n_groups, sms);
  return launch_kernel(k_backward_dw<T>, grid, smem, st, a);
}

template <typename T>
cudaError_t launch_backward_dx(const TailArgs& a, bool from_step, cudaStream_t st) {
  const size_t smem = smem_dx(sizeof(T), a.sh.k, a.sh.G, a.band);
  const int grid = (a.sh.Bp / 128) * a.n_bands * a.n_chunks;
  if (from_step) return launch_kernel(k_backward_dx<T, true>, grid, smem, st, a);
  return launch_kernel(k_backward_dx<T, false>, grid, smem, st, a);
}

cudaError_t launch_dx_reduce(const float* P, float* dX, int C, int d, int Bp, int B, int accumulate,
                             cudaStream_t st, const float* loss_part = nullptr, int n_loss = 0,
                             float scale = 0.f, float* loss = nullptr) {
  dim3 grid((d + 7) / 8, Bp / 128);
  k_dx_reduce<<<grid, 256, 0, st>>>(P, dX, C, d, Bp, B, accumulate, loss_part, n_loss, scale, loss);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_step(const TailArgs& a, int grid, cudaStream_t st) {
  const size_t smem = smem_step(sizeof(T), a.sh.k, a.sh.G, a.sh.Bp);
  return launch_kernel(k_step<T>, grid, smem, st, a);
}

template <typename T>
int step_grid(const TailArgs& a, int sms) {
  const size_t smem = smem_step(sizeof(T), a.sh.k, a.sh.G, a.sh.Bp);
  if (cudaFuncSetAttribute(k_step<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return 0;
  return resident_grid<T>((const void*)k_step<T>, smem, a.sh.n_groups, sms);
}

cudaError_t launch_loss_reduce(const float* part, int n, float scale, float* loss, cudaStream_t st) {
  k_loss_reduce<<<1, 32, 0, st>>>(part, n, scale, loss);
  return cudaGetLastError();
}

template cudaError_t launch_xt<float>(const void*, void*, int, int, int, cudaStream_t);
template cudaError_t launch_xt<__nv_bfloat16>(const void*, void*, int, int, int, cudaStream_t);
template cudaError_t launch_forward<float>(const TailArgs&, int, cudaStream_t);
template cudaError_t launch_forward<__nv_bfloat16>(const TailArgs&, int, cudaStream_t);
template cudaError_t launch_backward_dw<float>(const TailArgs&, int, cudaStream_t);
template cudaError_t launch_backward_dw<__nv_bfloat16>(const TailArgs&, int, cudaStream_t);
template cudaError_t launch_backward_dx<float>(const TailArgs&, bool, cudaStream_t);
template cudaError_t launch_backward_dx<__nv_bfloat16>(const TailArgs&, bool, cudaStream_t);
template cudaError_t launch_step<float>(const TailArgs&, int, cudaStream_t);
template cudaError_t launch_step<__nv_bfloat16>(const TailArgs&, int, cudaStream_t);
template int step_grid<float>(const TailArgs&, int);
template int step_grid<__nv_bfloat16>(const TailArgs&, int);

}  // namespace tail
}  // namespace haste
