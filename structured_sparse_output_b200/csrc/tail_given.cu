// tail_given.cu -- pipelined bf16 forward and dW of the group-shared sparse tail
// with a caller-provided upstream gradient (HASTE, "Hardware-Aware Dynamic Sparse
// Training for Large Output Spaces", Methodology 1: the G labels of a group read
// the same k gathered features, so each group is one dense product).  Up to four
// 128-row batch tiles (B <= 512).
//
// k_fwd3 -- one CTA per (group chunk, batch tile):
//   warps 0-3  producers: the gathered tile X[b-tile, I_g] (k rows of X^T, 128
//              batch columns) and the G x k weight block, cp.async into a ring;
//              warps 0 and 2 fill the even items, 1 and 3 the odd ones;
//   warp 4     MMA: logits tile (M = 128 batch rows, N = G, K = k) into a 2-deep
//              TMEM ring;
//   warps 5-8  epilogue: thread = batch row; the G logits of its row, as bf16, into
//              a shared-memory staging tile; each warp writes its 32 rows to
//              global memory with one TMA store (logits rows are L apart, so
//              per-thread stores would touch 32 rows per instruction).
// k_dw3 -- one CTA per group chunk, every batch row; items are (group, batch tile):
//   warps 0-3  producers: the gathered tile of the item and its dY tile (128 rows
//              x G, rows past B read as zeros), cp.async into a ring;
//   warp 4     MMA: dW_g^T (M = k slots, N = G, K = 128 batch rows of the item),
//              accumulated over the group's batch tiles in a 2-deep TMEM ring;
//   warps 5-8  epilogue: thread = slot; the group's dW columns as bf16.

#include "tail.cuh"

namespace haste {
namespace v3 {

using v2::publish_all;
using v2::wait_or_abort;

struct GivenArgs {
  TailShape sh;
  const int32_t* idx;
  const __nv_bfloat16* Xt;  // [d, Bp]
  const __nv_bfloat16* W;   // forward: [L, k]
  const __nv_bfloat16* dY;  // dW: [B, L]
  __nv_bfloat16* out;       // forward: logits [B, L]; dW: dW [L, k]
  int n_chunks, ns;
};

constexpr int kGivenThreads = 32 * 9;  // 4 producer warps, MMA warp, 4 epilogue warps
constexpr int kGivenMaxStages = 6;

// Shared memory: ns stages of (gathered tile [2 b-blocks][k rows + pad][128 B],
// second operand: weight block [k/64][G][128 B] (forward) or dY tile
// [128][2G B] (dW)), for the forward two staging tiles of the output
// [128][2G B], then the barriers.
struct GivenLayout {
  uint32_t xg_stride, op_stride, out_stride, xg, op, out, bars, total;
};
__host__ __device__ inline GivenLayout given_layout(int k, int G, int ns, bool fwd) {
  GivenLayout L;
  // 2 b-blocks of k rows; rows k..127 of the last block are padding that an
  // M = 128 product reads when k = 64 (those TMEM lanes are not read out)
  L.xg_stride = (uint32_t)((2 * k * 128 + (k < 128 ? (128 - k) * 128 : 0) + 1023) & ~1023);
  const uint32_t wb = (uint32_t)((k / 64) * G * 128), dyb = (uint32_t)(128 * G * 2);
  L.op_stride = ((wb > dyb ? wb : dyb) + 1023u) & ~1023u;
  uint32_t off = 0;
  L.xg = off;
  off += ns * L.xg_stride;
  L.op = off;
  off += ns * L.op_stride;
  L.out_stride = fwd ? (uint32_t)((128 * G * 2 + 1023) & ~1023) : 0u;
  L.out = off;
  off += 2 * L.out_stride;
  L.bars = off;
  off += 256;
  L.total = off + 1024;
  return L;
}

// cp.async of the gathered tile: rows idx_row[0..k) of X^T, batch columns
// [b0, b0 + 128), swizzled; the producer warp `part` (0 or 1) of a pair copies
// every other group of four rows.  Lane (rg, sub) copies 16-byte chunk sub of
// both 128-byte segments of its rows.
template <int kK>
__device__ __forceinline__ void gather_tile(uint32_t xg, const __nv_bfloat16* __restrict__ Xt, int Bp, int b0,
                                            const int (&rows_idx)[kK / 8], int part, int lane) {
  const int sub = lane & 7, rg = lane >> 3;
#pragma unroll
  for (int m = 0; m < kK / 8; ++m) {
    const int sl = rg + 4 * (m * 2 + part);
    const __nv_bfloat16* src = Xt + (int64_t)rows_idx[m] * Bp + b0 + sub * 8;
    const uint32_t dst = xg + sw128((uint32_t)(sl * 128 + sub * 16));
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) cp_async16(dst + (uint32_t)(bb * kK * 128), src + bb * 64, 16);
  }
}

template <int kK>
__device__ __forceinline__ void load_rows(int (&rows_idx)[kK / 8], const int32_t* __restrict__ idx, int64_t g,
                                          int part, int lane) {
  const int rg = lane >> 3;
#pragma unroll
  for (int m = 0; m < kK / 8; ++m) rows_idx[m] = idx[g * kK + rg + 4 * (m * 2 + part)];
}

// ============================================================ k_fwd3
template <int kG, int kK>
__global__ void __launch_bounds__(kGivenThreads, 1) k_fwd3(GivenArgs a, const __grid_constant__ CUtensorMap tm_out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TailShape sh = a.sh;
  const int NS = a.ns;
  const int n_bt = sh.Bp / 128;
  const int c = blockIdx.x / n_bt, t = blockIdx.x % n_bt;
  const int64_t gb = (int64_t)c * sh.n_groups / a.n_chunks;
  const int n_items = (int)((int64_t)(c + 1) * sh.n_groups / a.n_chunks - gb);
  const GivenLayout Lo = given_layout(kK, kG, NS, true);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;                        // [NS] stage loaded (count: the two producer warps of the item)
  uint64_t* empty = full + kGivenMaxStages;     // [NS] stage read by the MMA
  uint64_t* f_full = empty + kGivenMaxStages;   // [2] logits in TMEM
  uint64_t* f_empty = f_full + 2;               // [2] logits read out (4 epilogue warps)
  uint64_t* done = f_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 64);
      mbar_init(&empty[st], 1);
    }
    for (int z = 0; z < 2; ++z) {
      mbar_init(&f_full[z], 1);
      mbar_init(&f_empty[z], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t ncols = tmem_cols_for(2 * kG);
  if (w == 4) {
    tmem_alloc(tslot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  auto XG = [&](int st) -> uint32_t { return base + Lo.xg + st * Lo.xg_stride; };
  auto OP = [&](int st) -> uint32_t { return base + Lo.op + st * Lo.op_stride; };

  if (w < 4) {
    // ------------------------------------------------------------ producers
    const int half = w & 1, part = w >> 1;
    for (int i = half; i < n_items; i += 2) {
      const int64_t g = gb + i;
      const int st = i % NS;
      int rows_idx[kK / 8];
      load_rows<kK>(rows_idx, a.idx, g, part, lane);
      if (!wait_or_abort(&empty[st], ((i / NS) & 1) ^ 1, abort_flag)) break;
      gather_tile<kK>(XG(st), a.Xt, sh.Bp, t * 128, rows_idx, part, lane);
      // weight block (contiguous G x k), chunks split between the pair
      const __nv_bfloat16* wsrc = a.W + g * (int64_t)kG * kK;
      constexpr int cpr = kK / 8;
#pragma unroll 4
      for (int c0 = 32 * part; c0 < kG * cpr; c0 += 64) {
        const int cc = c0 + lane;
        const int j = cc / cpr, q = cc % cpr;
        cp_async16(OP(st) + sw128((uint32_t)((q >> 3) * kG * 128 + j * 128 + (q & 7) * 16)),
                   wsrc + (int64_t)j * kK + q * 8, 16);
      }
      cp_async_commit();
      publish_all(&full[st]);
    }
    cp_async_wait_all();
  } else if (w == 4) {
    // ------------------------------------------------------------------ MMA
    const uint32_t idesc = make_idesc(1, 1, 0, 128, kG);  // A MN-major (batch contiguous), B K-major
    for (int i = 0; i < n_items; ++i) {
      const int st = i % NS, fb = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&f_empty[fb], ((i >> 1) & 1) ^ 1, abort_flag))) break;
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[st], (i / NS) & 1, abort_flag))) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < kK / 16; ++kk) {
          const uint64_t ad = make_sdesc(XG(st) + (uint32_t)(kk * 16 * 128), (uint32_t)kK * 128, 1024, kLayoutSw128);
          const uint64_t bd =
              make_sdesc(OP(st) + (uint32_t)((kk / 4) * kG * 128 + (kk % 4) * 32), 16, 1024, kLayoutSw128);
          mma_ss<false>(tmem + (uint32_t)(fb * kG), ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&f_full[fb]);
        mma_commit(&empty[st]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(done);  // also after an abort: TMEM is freed only once the MMAs end
    __syncwarp();
    (void)__all_sync(0xffffffffu, mbar_wait(done, 0));
  } else {
    // ------------------------------------------------------------- epilogue
    constexpr int RB = kG * 2;  // bytes of an output row
    const int q = w & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int r = q * 32 + lane;                      // row of the batch tile
    const bool warp_rows = t * 128 + q * 32 < sh.B;  // some of this warp's rows are inside the batch
    for (int i = 0; i < n_items; ++i) {
      const int fb = i & 1;
      // this warp's store from the same staging tile two items ago has read it
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      if (!__all_sync(0xffffffffu, wait_or_abort(&f_full[fb], (i >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      float vall[kG];
#pragma unroll
      for (int c0 = 0; c0 < kG; c0 += 16)
        tmem_ld16(tmem + lane_off + (uint32_t)(fb * kG + c0), *reinterpret_cast<float(*)[16]>(&vall[c0]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&f_empty[fb]);  // TMEM read: the next product may overwrite it
      uint8_t* out = gbase + Lo.out + fb * Lo.out_stride;
#pragma unroll
      for (int c0 = 0; c0 < kG; c0 += 8) {
        const float* v = &vall[c0];
        const uint4 pk = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                    pack_bf16x2(v[6], v[7]));
        *reinterpret_cast<uint4*>(out + swz_rows((uint32_t)(r * RB + c0 * 2), RB)) = pk;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && warp_rows) {
        tma_store_2d(&tm_out, base + Lo.out + fb * Lo.out_stride + (uint32_t)(q * 32 * RB), (int)((gb + i) * kG),
                     t * 128 + q * 32);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();  // the stores are complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (w == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// ============================================================= k_dw3
template <int kG, int kK>
__global__ void __launch_bounds__(kGivenThreads, 1) k_dw3(GivenArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int RB = kG * 2;  // bytes of a dY row
  const TailShape sh = a.sh;
  const int NS = a.ns;
  const int n_bt = sh.Bp / 128;
  const int64_t gb = (int64_t)blockIdx.x * sh.n_groups / a.n_chunks;
  const int n_groups = (int)((int64_t)(blockIdx.x + 1) * sh.n_groups / a.n_chunks - gb);
  const int n_items = n_groups * n_bt;  // item i: group i / n_bt, batch tile i % n_bt
  const GivenLayout Lo = given_layout(kK, kG, NS, false);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;
  uint64_t* empty = full + kGivenMaxStages;
  uint64_t* d_full = empty + kGivenMaxStages;  // [2] a group's dW in TMEM
  uint64_t* d_empty = d_full + 2;              // [2] read out (4 epilogue warps)
  uint64_t* done = d_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 64);
      mbar_init(&empty[st], 1);
    }
    for (int z = 0; z < 2; ++z) {
      mbar_init(&d_full[z], 1);
      mbar_init(&d_empty[z], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t ncols = tmem_cols_for(2 * kG);
  if (w == 4) {
    tmem_alloc(tslot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  auto XG = [&](int st) -> uint32_t { return base + Lo.xg + st * Lo.xg_stride; };
  auto OP = [&](int st) -> uint32_t { return base + Lo.op + st * Lo.op_stride; };

  if (w < 4) {
    // ------------------------------------------------------------ producers
    const int half = w & 1, part = w >> 1;
    for (int i = half; i < n_items; i += 2) {
      const int64_t g = gb + i / n_bt;
      const int t = i % n_bt, st = i % NS;
      int rows_idx[kK / 8];
      load_rows<kK>(rows_idx, a.idx, g, part, lane);
      if (!wait_or_abort(&empty[st], ((i / NS) & 1) ^ 1, abort_flag)) break;
      gather_tile<kK>(XG(st), a.Xt, sh.Bp, t * 128, rows_idx, part, lane);
      // dY tile: 128 rows of 2G bytes (rows at or past B read as zeros), swizzled by row width
      constexpr int cpr = RB / 16;
      for (int c0 = 32 * part; c0 < 128 * cpr; c0 += 64) {
        const int cc = c0 + lane;
        const int r = cc / cpr, q = cc % cpr;
        const int b = t * 128 + r;
        const bool in = b < sh.B;
        const __nv_bfloat16* src = in ? a.dY + (int64_t)b * sh.L + g * kG + q * 8 : a.dY;
        cp_async16(OP(st) + swz_rows((uint32_t)(r * RB + q * 16), RB), src, in ? 16u : 0u);
      }
      cp_async_commit();
      publish_all(&full[st]);
    }
    cp_async_wait_all();
  } else if (w == 4) {
    // ------------------------------------------------------------------ MMA
    const uint32_t idesc = make_idesc(1, 0, 1, 128, kG);  // A K-major (X_g^T), B MN-major (dY)
    bool ok = true;
    for (int i = 0; ok && i < n_items; ++i) {
      const int gi = i / n_bt, t = i % n_bt, st = i % NS, db = gi & 1;
      if (t == 0 && !__all_sync(0xffffffffu, wait_or_abort(&d_empty[db], ((gi >> 1) & 1) ^ 1, abort_flag))) break;
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[st], (i / NS) & 1, abort_flag))) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int b = kk * 16;
          const uint64_t ad =
              make_sdesc(XG(st) + (uint32_t)((b / 64) * kK * 128 + (kk % 4) * 32), 16, 1024, kLayoutSw128);
          const uint64_t bd = make_sdesc(OP(st) + (uint32_t)(b * RB), 16, 8 * RB, layout_for_rows(RB));
          mma_ss<false>(tmem + (uint32_t)(db * kG), ad, bd, idesc, (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[st]);
        if (t == n_bt - 1) mma_commit(&d_full[db]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(done);
    __syncwarp();
    (void)__all_sync(0xffffffffu, mbar_wait(done, 0));
  } else {
    // ------------------------------------------------------------- epilogue
    const int q = w & 3;
    const int r = q * 32 + lane;  // slot
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    for (int gi = 0; gi < n_groups; ++gi) {
      const int db = gi & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&d_full[db], (gi >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const int64_t g = gb + gi;
      float vall[kG];
#pragma unroll
      for (int c0 = 0; c0 < kG; c0 += 16)
        tmem_ld16(tmem + lane_off + (uint32_t)(db * kG + c0), *reinterpret_cast<float(*)[16]>(&vall[c0]));
      tmem_wait_ld();
#pragma unroll
      for (int c0 = 0; c0 < kG; c0 += 16) {
        const float* v = &vall[c0];
        if (r < kK) {
          __nv_bfloat16* dst = a.out + (g * kG + c0) * kK + r;  // lanes: consecutive slots
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[(int64_t)e * kK] = __float2bfloat16_rn(v[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[db]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace v3

// ------------------------------------------------------------- host side
namespace tail3 {

bool supported(int G, int k, int Bp) {
  return (G == 16 || G == 32 || G == 64) && (k == 64 || k == 128) && Bp <= 512;
}

size_t smem_for(int k, int G, int ns, bool fwd) { return v3::given_layout(k, G, ns, fwd).total; }

// Deepest ring (2 to 6 stages) that fits; 0 when two stages do not.
int stages(int k, int G, size_t smem_optin, size_t reserve, bool fwd) {
  int best = 0;
  for (int st = 2; st <= v3::kGivenMaxStages; ++st)
    if (smem_for(k, G, st, fwd) + reserve <= smem_optin) best = st;
  return best;
}

template <int kG, int kK>
cudaError_t launch_fwd_t(const v3::GivenArgs& a, cudaStream_t st) {
  const size_t smem = smem_for(kK, kG, a.ns, true);
  auto kern = v3::k_fwd3<kG, kK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // the logits [B, L] as the stores' tensor: boxes of G labels x 32 rows
  CUtensorMap tm_out;
  e = tail2::tmap_2d(&tm_out, a.out, (uint64_t)a.sh.L, (uint64_t)a.sh.B, (uint64_t)a.sh.L * 2, kG, 32);
  if (e != cudaSuccess) return e;
  kern<<<a.n_chunks * (a.sh.Bp / 128), v3::kGivenThreads, smem, st>>>(a, tm_out);
  return cudaGetLastError();
}

template <int kG, int kK>
cudaError_t launch_dw_t(const v3::GivenArgs& a, cudaStream_t st) {
  const size_t smem = smem_for(kK, kG, a.ns, false);
  auto kern = v3::k_dw3<kG, kK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<a.n_chunks, v3::kGivenThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int G, int k, const v3::GivenArgs& a, cudaStream_t st) {
  HASTE_V2_DISPATCH(launch_fwd_t, a, st)
}
cudaError_t launch_dw(int G, int k, const v3::GivenArgs& a, cudaStream_t st) {
  HASTE_V2_DISPATCH(launch_dw_t, a, st)
}

}  // namespace tail3
}  // namespace haste
