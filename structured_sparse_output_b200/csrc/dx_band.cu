// dx_band.cu -- dX of the group-shared sparse tail as dense band products
// (HASTE, "Hardware-Aware Dynamic Sparse Training for Large Output Spaces",
// Methodology 1; the dX step of the backward pass).
//
// k_dx_band -- per CTA (feature band, group chunk, batch half of up to 256 rows):
//   warp 0 loads each ring item's dY tile and weight rows into a shared-memory
//   ring with TMA, warps 2-9 (two sets of four, alternate items) densify the
//   weight rows over the band, warp 1 issues the item's MMAs per 128-row batch
//   tile into TMEM accumulators, and warps 2-9 write the chunk partial at the end.
//   k_dx_reduce (tail.cu) sums the chunk partials in order.
//
// A ring item is a super-group: NG = 64 / G consecutive groups, 64 labels.  Its
// dY columns and weight rows are contiguous (row-major dY [B, L], W [L, k]; the
// fused step writes its gradient buffer transposed, as label rows [n_items * 64]
// [Bp]), so a few TMA boxes per operand carry the whole item, with rows of 128
// bytes, and one item's MMA chain has K = 64 whatever G: groups of 16 or 32
// labels cost the ring round trip of one group of 64.

#include "tail.cuh"

namespace haste {
namespace v2 {

struct DxArgs {
  TailShape sh;
  const int32_t* idx;
  const __nv_bfloat16* dY;  // for L2 prefetches of the fused step's buffer
  const __nv_bfloat16* W;
  float* dX_part;
  int band, n_bands, n_chunks, ns;  // ns: stages of the shared-memory ring
  int n_halves;                      // batch halves of up to 256 rows (2 when B > 256)
  int group_major;                   // dY is the fused step's buffer [n_items * 64][Bp], else [B, L]
};

constexpr int kMaxDxStages = 6;  // deepest ring of the dX pass
constexpr int kDxPrefetch = 8;   // items ahead of the ring loads that are prefetched into L2
constexpr int kItemLabels = 64;  // labels of a ring item (a super-group)

// Groups per ring item, and the number of items (super-groups) of n_groups groups.
__host__ __device__ constexpr int items_ng(int G) { return kItemLabels / G; }
__host__ __device__ inline int64_t n_items_of(int64_t n_groups, int G) {
  return (n_groups + items_ng(G) - 1) / items_ng(G);
}

struct DxLayout {
  uint32_t dy, wt, bars, total, dy_stride, wt_stride;
};
// Shared memory of the dX pass: ns stages of (dY tile [rows][64], densified weight
// block [band][64]; 128-byte rows, 128B swizzle) and the barriers.  The weight
// rows are read by the densify warps straight from global memory (L2), so that a
// third stage fits.
__host__ __device__ inline DxLayout dx_layout(int rows, int band, int k, int ns) {
  (void)k;
  DxLayout L;
  L.dy_stride = (uint32_t)((rows * 128 + 1023) & ~1023);
  L.wt_stride = (uint32_t)((band * 128 + 1023) & ~1023);
  uint32_t off = 0;
  L.dy = off;
  off += ns * L.dy_stride;
  L.wt = off;
  off += ns * L.wt_stride;
  L.bars = off;
  off += 512;
  L.total = off + 1024;
  return L;
}

// ========================================================== k_dx_band
constexpr int kDxThreads = 320;  // producer warp, MMA warp, two sets of 4 densify / epilogue warps

// The dX pass as one dense product per item and feature band.  For a band of NB
// features [f0, f0+NB), the densified weight block Wt_u[n][c] (n over the band,
// c over the item's 64 labels, group j of the item owning columns [jG, jG+G))
// holds W[g_j*G + c - jG, s] in the row of the feature f0 + n = idx[g_j][s] and
// zeros elsewhere; then
//   dX[b, f0 + n] = sum over items u (ascending) of sum_c dY[b, 64u + c] Wt_u[n][c],
// MMAs per 128-row batch tile (M = 128 batch rows, N = NB, K = 16 per
// instruction) over the item's present labels, accumulated in TMEM.  A group's
// slots hold distinct features, so a (b, f) entry receives exactly group g_j's
// term dY_g[b, :] . W_g[:, s] for every group of the item, in ascending order.
// One CTA owns a feature band, a batch half of up to 256 rows (up to two 128-row
// TMEM accumulators of NB columns) and a chunk of whole items:
//   producer (warp 0, one thread): the item's dY tile (the half's rows x 64
//     labels) into a ring stage, and the item's weight rows and index rows into
//     L2 ahead of use;
//   densify (two sets of four warps, warps 2-5 for the even items of the chunk,
//     6-9 for the odd ones; the thread of slot s): loads column s of each present
//     group's weights from global memory when the slot's feature falls in the
//     band (the lanes of a warp read consecutive slots of one weight row), clears,
//     for each group of the item NS back (the previous user of the stage), that
//     group's columns of the Wt row of its slot's feature, then, after a barrier
//     of its set, writes the loaded column into the group's columns of the row
//     of the slot's feature;
//   MMA (warp 1): D[t] += dY_u[128t.., labels] . Wt_u^T for each batch tile t;
//   epilogue (warps 2-9): the TMEM accumulators to the chunk partial.
// The warps of a set run the same number of iterations (one per item of the
// set), so its named barrier always matches; a wait that runs out raises the
// abort flag and the remaining iterations skip their work.
template <int kG, int kK>
__global__ void __launch_bounds__(kDxThreads, 1)
    k_dx_band(DxArgs a, const __grid_constant__ CUtensorMap tm_dy) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int NG = items_ng(kG);  // groups per item
  constexpr int GB = kG * 2;        // bytes of one group's columns in a 128-byte row
  const int NS = a.ns, NB = a.band;
  const TailShape sh = a.sh;
  const int BH = min(sh.Bp, 256);  // rows of the dY box (a batch half)
  const int h = blockIdx.x % a.n_bands;
  const int bh = (blockIdx.x / a.n_bands) % a.n_halves;
  const int c = blockIdx.x / (a.n_bands * a.n_halves);
  const int MT = min(2, (sh.Bp - 256 * bh) / 128);  // 128-row tiles of this half
  const int f0 = h * NB;
  const int nf = min(sh.d, f0 + NB) - f0;
  const int64_t n_sg = n_items_of(sh.n_groups, kG);
  const int64_t u0 = (int64_t)c * n_sg / a.n_chunks;
  const int64_t u1 = (int64_t)(c + 1) * n_sg / a.n_chunks;
  const int n = (int)(u1 - u0);  // items of the chunk
  // groups of item u of the chunk: [(u0 + u) * NG, ... + cnt(u))
  auto cnt = [&](int u) -> int { return (int)min((int64_t)NG, sh.n_groups - (u0 + u) * NG); };

  const DxLayout Lo = dx_layout(BH, NB, kK, NS);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  auto DYS = [&](int st) -> uint32_t { return base + Lo.dy + st * Lo.dy_stride; };
  auto WT = [&](int st) -> uint32_t { return base + Lo.wt + st * Lo.wt_stride; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;                      // [NS] dY tile landed (1 + tx bytes)
  uint64_t* empty = full + kMaxDxStages;      // [NS] dY tile read (MMA commit)
  uint64_t* wt_full = empty + kMaxDxStages;   // [NS] Wt block written (4 densify warps)
  uint64_t* wt_empty = wt_full + kMaxDxStages;  // [NS] Wt block read by the MMA
  uint64_t* done = wt_empty + kMaxDxStages;     // every MMA of the CTA finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int w = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);   // MMA commit
      mbar_init(&wt_full[st], 4);
      mbar_init(&wt_empty[st], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t tmem_cols = (uint32_t)MT * 256;
  if (w == 1) {
    tmem_alloc(tslot, tmem_cols);
    tmem_relinquish();
  }
  if (w >= 2) {
    // zero Wt blocks, no rows written yet
    const int t = threadIdx.x - 64;
    uint4* wt0 = reinterpret_cast<uint4*>(gbase + Lo.wt);
    for (uint32_t e = (uint32_t)t; e < (uint32_t)NS * Lo.wt_stride / 16; e += 256) wt0[e] = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (w == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t bytes = (uint32_t)BH * 128;  // dY tile (full boxes)
      const int64_t w_elems = sh.L * kK, ix_elems = sh.n_groups * kK;
      // a ring load from HBM takes longer than the ring's MMA work: the tiles of
      // later items are requested into L2 ahead of their ring loads (ranges clamped
      // to the tensors)
      auto prefetch = [&](int64_t sg) {
        if (a.group_major) prefetch_l2(a.dY + sg * kItemLabels * sh.Bp, (uint32_t)(kItemLabels * sh.Bp * 2));
        const int64_t w0 = sg * kItemLabels * kK, i0 = sg * NG * kK;
        prefetch_l2(a.W + w0, (uint32_t)(min((int64_t)kItemLabels * kK, w_elems - w0) * 2));
        prefetch_l2(a.idx + i0, (uint32_t)(min((int64_t)NG * kK, ix_elems - i0) * 4));
      };
      for (int i = 0; i < kDxPrefetch && i < n; ++i) prefetch(u0 + i);
      int st = 0, ph = 0, issued = 0;
      for (int i = 0; i < n; ++i) {
        const int64_t sg = u0 + i;
        if (i + kDxPrefetch < n) prefetch(sg + kDxPrefetch);
        if (!wait_or_abort(&empty[st], ph ^ 1, abort_flag)) break;
        ++issued;
        mbar_arrive_expect_tx(&full[st], bytes);
        if (a.group_major) {
          for (int blk = 0; blk < BH / 64; ++blk)
            tma_load_2d(DYS(st) + (uint32_t)(blk * 64 * 128), &tm_dy, 256 * bh + 64 * blk, (int)(sg * kItemLabels),
                        &full[st]);
        } else
          tma_load_2d(DYS(st), &tm_dy, (int)(sg * kItemLabels), 256 * bh, &full[st]);
        if (++st == NS) {
          st = 0;
          ph ^= 1;
        }
      }
      // no copy may still be landing when the CTA exits (an abort can leave the
      // last stages unconsumed)
      for (int j = issued > NS ? issued - NS : 0; j < issued; ++j) mbar_wait(&full[j % NS], (j / NS) & 1);
    }
  } else if (w == 1) {
    // ------------------------------------------------------------- MMA
    const uint32_t idesc = make_idesc(1, a.group_major ? 1u : 0u, 0, 128, (uint32_t)NB);
    int st = 0, ph = 0;
    for (int i = 0; i < n; ++i) {
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[st], ph, abort_flag))) break;
      if (!__all_sync(0xffffffffu, wait_or_abort(&wt_full[st], ph, abort_flag))) break;
      tc_fence_after();
      if (lane == 0) {
        const int nk = cnt(i) * (kG / 16);  // K steps of the item's present labels
        // the fused step's tile is label rows (batch contiguous: MN-major, 64-row
        // blocks 8 KB apart), a caller's is batch rows (labels contiguous: K-major);
        // descriptors advance by start-address offsets (16-byte units), so that an
        // MMA costs few instructions of this warp, which shares its scheduler with
        // densify warps
        const uint64_t ad0 = a.group_major ? make_sdesc(DYS(st), 64 * 128, 1024, kLayoutSw128)
                                           : make_sdesc(DYS(st), 16, 1024, kLayoutSw128);
        const uint32_t kstep = a.group_major ? 16 * 128 / 16 : 32 / 16;
        const uint64_t bd0 = make_sdesc(WT(st), 16, 1024, kLayoutSw128);
        for (int t = 0; t < MT; ++t)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (kk < nk)
              mma_ss<false>(tmem + (uint32_t)(t * 256), ad0 + (uint64_t)(t * 1024 + kk * kstep), bd0 + (uint64_t)(kk * 2),
                            idesc, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[st]);
        mma_commit(&wt_empty[st]);
      }
      __syncwarp();
      if (++st == NS) {
        st = 0;
        ph ^= 1;
      }
    }
    if (lane == 0) mma_commit(done);  // also after an abort: TMEM is freed only once the MMAs end
    __syncwarp();
  } else {
    // ----------------------------------------------- densify, then epilogue
    const int set = (w - 2) >> 2;          // items i = set, set + 2, ...
    const int s = (threadIdx.x - 64) & 127;  // this thread's slot
    const bool slot_ok = s < kK;
    const uint16_t* wbits = reinterpret_cast<const uint16_t*>(a.W);
    // the slot's feature in group j of item i, relative to the band (-1 if absent)
    auto feat = [&](int i, int j) -> int {
      if (!slot_ok || i < 0 || i >= n || j >= cnt(i)) return -1;
      return a.idx[((u0 + i) * NG + j) * kK + s] - f0;
    };
    // features of this set's next three items, and of the items NS before them
    // (the previous users of the same ring stages), loaded ahead
    int fa[NG], fb[NG], fc[NG], oa[NG], ob[NG], oc[NG];
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      fa[j] = feat(set, j);
      fb[j] = feat(set + 2, j);
      fc[j] = feat(set + 4, j);
      oa[j] = feat(set - NS, j);
      ob[j] = feat(set + 2 - NS, j);
      oc[j] = feat(set + 4 - NS, j);
    }
    // ring position of item i, advanced by two items per iteration (NS >= 2)
    int st = set;
    uint32_t ph = 0;
    for (int i = set; i < n; i += 2) {
      int fcur[NG], fold[NG];
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        fcur[j] = fa[j];
        fold[j] = oa[j];
        fa[j] = fb[j];
        fb[j] = fc[j];
        fc[j] = feat(i + 6, j);
        oa[j] = ob[j];
        ob[j] = oc[j];
        oc[j] = feat(i + 6 - NS, j);
      }
      // column s of the item's weights (label rows 64 (u0 + i) + j G + l), loaded
      // before the waits so that their latency hides behind them
      uint32_t pk[NG][kG / 2];
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        if (fcur[j] >= 0 && fcur[j] < nf) {
          const uint16_t* col = wbits + ((u0 + i) * kItemLabels + j * kG) * kK + s;
#pragma unroll
          for (int l = 0; l < kG; l += 2)
            pk[j][l / 2] = (uint32_t)__ldg(col + (int64_t)l * kK) | ((uint32_t)__ldg(col + (int64_t)(l + 1) * kK) << 16);
        }
      }
      uint8_t* wt = gbase + Lo.wt + st * Lo.wt_stride;
      // the MMA of item i - NS has read this stage's Wt block: clear its groups' columns
      const bool ok = __all_sync(0xffffffffu, wait_or_abort(&wt_empty[st], ph ^ 1u, abort_flag));
      if (ok) {
#pragma unroll
        for (int j = 0; j < NG; ++j)
          if (fold[j] >= 0 && fold[j] < nf) {
#pragma unroll
            for (int cc = 0; cc < GB / 16; ++cc)
              *reinterpret_cast<uint4*>(wt + sw128((uint32_t)(fold[j] * 128 + j * GB + cc * 16))) =
                  make_uint4(0, 0, 0, 0);
          }
      }
      // every old column run is clear before any new one is written (slots of
      // different items may share a feature)
      named_bar(1 + set, 128);
      if (ok) {
#pragma unroll
        for (int j = 0; j < NG; ++j) {
          const int f = fcur[j];
          if (f < 0 || f >= nf) continue;
#pragma unroll
          for (int cc = 0; cc < GB / 16; ++cc)
            *reinterpret_cast<uint4*>(wt + sw128((uint32_t)(f * 128 + j * GB + cc * 16))) =
                make_uint4(pk[j][4 * cc], pk[j][4 * cc + 1], pk[j][4 * cc + 2], pk[j][4 * cc + 3]);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&wt_full[st]);
      if ((st += 2) >= NS) {
        st -= NS;
        ph ^= 1u;
      }
    }
    // ------------------------------------------------------------ epilogue
    const bool fin = __all_sync(0xffffffffu, mbar_wait(done, 0)) && !*abort_flag;
    tc_fence_after();
    const int q = w & 3;  // TMEM lane quarter: batch rows 32q.. of each tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    if (fin) {
      // two batch tiles: one per set; one tile: the sets take alternate 16-column chunks
      for (int t = MT == 2 ? set : 0; t < (MT == 2 ? set + 1 : 1); ++t) {
        const int b = 256 * bh + t * 128 + q * 32 + lane;
        for (int c0 = MT == 2 ? 0 : 16 * set; c0 < NB; c0 += MT == 2 ? 16 : 32) {
          float v[16];
          tmem_ld16(tmem + lane_off + (uint32_t)(t * 256 + c0), v);
          tmem_wait_ld();
          float* dst = a.dX_part + ((int64_t)c * sh.d + f0 + c0) * sh.Bp + b;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c0 + e < nf) dst[(int64_t)e * sh.Bp] = n > 0 ? v[e] : 0.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace v2

// ------------------------------------------------------------- host side
namespace tail2 {

bool dx_supported(int G, int k, int Bp) {
  return (G == 16 || G == 32 || G == 64) && (k == 64 || k == 128) && Bp <= 512;
}

size_t dx_smem(int rows, int band, int k, int ns) { return v2::dx_layout(rows, band, k, ns).total; }

// Feature bands and ring depth of the dX pass: bands of at most 256 features
// (the widest MMA N), as few as cover d, split evenly in multiples of 16; the
// deepest ring (up to six stages) that fits in the shared memory left after
// `reserve` bytes.  Returns false when two stages do not fit.
bool dx_config(int G, int k, int d, int Bp, size_t smem_optin, size_t reserve, int* band, int* n_bands, int* ns) {
  (void)G;
  const int rows = Bp < 256 ? Bp : 256;  // a CTA covers a batch half of up to 256 rows
  const int nb = (d + 255) / 256;
  const int bw = (((d + nb - 1) / nb) + 15) & ~15;
  int best = 0;
  for (int st = 2; st <= v2::kMaxDxStages; ++st)
    if (dx_smem(rows, bw, k, st) + reserve <= smem_optin) best = st;
  if (!best) return false;
  *band = bw;
  *n_bands = nb;
  *ns = best;
  return true;
}

// Items (super-groups of 64 labels) of the dX pass for n_groups groups of G.
int64_t dx_items(int64_t n_groups, int G) { return v2::n_items_of(n_groups, G); }

// dY of the dX pass, either the fused step's buffer of label rows [n_items * 64]
// [Bp] (columns past B hold zeros) or a caller's row-major [B, L] (rows past B are
// outside the tensor and read as zeros).
template <int kG, int kK>
cudaError_t launch_dx_t(v2::DxArgs a, const void* dY, const void* W, cudaStream_t st) {
  (void)W;  // the densify warps read a.W directly
  const int rows = a.sh.Bp < 256 ? a.sh.Bp : 256;
  const size_t smem = dx_smem(rows, a.band, kK, a.ns);
  auto kern = v2::k_dx_band<kG, kK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_dy;
  if (a.group_major)
    e = tmap_2d(&tm_dy, dY, (uint64_t)a.sh.Bp, (uint64_t)dx_items(a.sh.n_groups, kG) * v2::kItemLabels,
                (uint64_t)a.sh.Bp * 2, 64, v2::kItemLabels);
  else
    e = tmap_2d(&tm_dy, dY, (uint64_t)a.sh.L, (uint64_t)a.sh.B, (uint64_t)a.sh.L * 2, v2::kItemLabels,
                (uint32_t)rows);
  if (e != cudaSuccess) return e;
  const int grid = a.n_bands * a.n_halves * a.n_chunks;
  kern<<<grid, v2::kDxThreads, smem, st>>>(a, tm_dy);
  return cudaGetLastError();
}

cudaError_t launch_dx(int G, int k, const v2::DxArgs& a, const void* dY, const void* W, cudaStream_t st) {
  HASTE_V2_DISPATCH(launch_dx_t, a, dY, W, st)
}

}  // namespace tail2
}  // namespace haste
