// dx_band.cu -- dX of the group-shared sparse tail as dense band products
// (HASTE, "Hardware-Aware Dynamic Sparse Training for Large Output Spaces",
// Methodology 1; the dX step of the backward pass).
//
// k_dx_band -- per CTA (feature band, group chunk, batch half of up to 256 rows): warp 0 loads
//   each group's dY tile and G x k weight block into a shared-memory ring with
//   TMA, warps 2-9 (two sets of four, alternate groups) densify the weight block
//   over the band, warp 1 issues one MMA per 128-row batch tile into TMEM
//   accumulators, and warps 2-9 write the chunk partial at the end.  k_dx_reduce
//   (tail.cu) sums the chunk partials in order.

#include "tail.cuh"

namespace haste {
namespace v2 {

struct DxArgs {
  TailShape sh;
  const int32_t* idx;
  const __nv_bfloat16* dY;  // for L2 prefetches of the group-major buffer
  const __nv_bfloat16* W;
  float* dX_part;
  int band, n_bands, n_chunks, ns;  // ns: stages of the shared-memory ring
  int n_halves;                      // batch halves of up to 256 rows (2 when B > 256)
  // element (b, g*G + j) of dY is at dY[g*dy_gstride + b*dy_rstride + j]
  int64_t dy_gstride, dy_rstride;
  // dY tile of group g (the batch half's rows) in the dY tensor map: x = g*dy_xg,
  // y = g*dy_yg + 256*half
  int dy_xg, dy_yg;
};

constexpr int kMaxDxStages = 6;  // deepest ring of the dX pass
constexpr int kDxPrefetch = 8;   // groups ahead of the ring loads that are prefetched into L2

struct DxLayout {
  uint32_t dy, w, wt, bars, total, dy_stride, w_stride, wt_stride;
};
// Shared memory of the dX pass: ns stages of (dY tile [Bp][G], weight block
// [k/64][G][64], densified weight block [band][G]) and the barriers.
__host__ __device__ inline DxLayout dx_layout(int Bp, int band, int k, int G, int ns) {
  DxLayout L;
  L.dy_stride = (uint32_t)((Bp * G * 2 + 1023) & ~1023);
  L.w_stride = (uint32_t)(((k / 64) * G * 128 + 1023) & ~1023);
  L.wt_stride = (uint32_t)((band * G * 2 + 1023) & ~1023);
  uint32_t off = 0;
  L.dy = off;
  off += ns * L.dy_stride;
  L.w = off;
  off += ns * L.w_stride;
  L.wt = off;
  off += ns * L.wt_stride;
  L.bars = off;
  off += 512;
  L.total = off + 1024;
  return L;
}

// ========================================================== k_dx_band
constexpr int kDxThreads = 320;  // producer warp, MMA warp, two sets of 4 densify / epilogue warps

// The dX pass as one dense product per group and feature band.  For a band of
// NB features [f0, f0+NB), the densified weight block Wt_g[n][j'] (n over the
// band, j' over the G labels of group g) holds W[g*G + j', s] in the row of the
// feature f0 + n = idx[g][s] and zeros elsewhere; then
//   dX[b, f0 + n] = sum over groups g (ascending) of sum_j' dY[b, g*G + j'] Wt_g[n][j'],
// one tcgen05 MMA per 128-row batch tile and group (M = 128 batch rows, N = NB,
// K = G), accumulated in TMEM.  A group's slots hold distinct features, so a
// (b, f) entry receives exactly that group's term dY_g[b, :] . W_g[:, s].
// One CTA owns a feature band, a batch half of up to 256 rows (up to two 128-row
// TMEM accumulators of NB columns) and a chunk of groups:
//   producer (warp 0, one thread): the dY tile (Bp x G, K-major, swizzled rows of
//     2G bytes) and the G x k weight block into a stage of the ring with TMA;
//   densify (two sets of four warps, warps 2-5 for the even groups of the chunk,
//     6-9 for the odd ones; the thread of slot s): clears the Wt row of slot s's
//     feature in group i - NS (the previous user of the stage, read from the
//     index array), then, after a barrier of its set, copies column s of the
//     weight block into the Wt row of the slot's feature when it falls in the
//     band;
//   MMA (warp 1): D[t] += dY_g[128t.., :] . Wt_g^T for each batch tile t;
//   epilogue (warps 2-9): the TMEM accumulators to the chunk partial.
// The warps of a set run the same number of iterations (one per group of the
// set), so its named barrier always matches; a wait that runs out raises the
// abort flag and the remaining iterations skip their work.
template <int kG, int kK>
__global__ void __launch_bounds__(kDxThreads, 1)
    k_dx_band(DxArgs a, const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int RB = kG * 2;  // bytes of a K-major row (G bf16)
  const int NS = a.ns, NB = a.band;
  const TailShape sh = a.sh;
  const int BH = min(sh.Bp, 256);  // rows of the dY box (a batch half)
  const int h = blockIdx.x % a.n_bands;
  const int bh = (blockIdx.x / a.n_bands) % a.n_halves;
  const int c = blockIdx.x / (a.n_bands * a.n_halves);
  const int MT = min(2, (sh.Bp - 256 * bh) / 128);  // 128-row tiles of this half
  const int f0 = h * NB;
  const int nf = min(sh.d, f0 + NB) - f0;
  const int64_t g0 = (int64_t)c * sh.n_groups / a.n_chunks;
  const int64_t g1 = (int64_t)(c + 1) * sh.n_groups / a.n_chunks;
  const int n = (int)(g1 - g0);

  const DxLayout Lo = dx_layout(BH, NB, kK, kG, NS);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  auto DYS = [&](int st) -> uint32_t { return base + Lo.dy + st * Lo.dy_stride; };
  auto WS = [&](int st) -> uint32_t { return base + Lo.w + st * Lo.w_stride; };
  auto WT = [&](int st) -> uint32_t { return base + Lo.wt + st * Lo.wt_stride; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;                      // [NS] dY tile + weight block landed (1 + tx bytes)
  uint64_t* empty = full + kMaxDxStages;      // [NS] both read: MMA commit + 4 densify warps
  uint64_t* wt_full = empty + kMaxDxStages;   // [NS] Wt block written (4 densify warps)
  uint64_t* wt_empty = wt_full + kMaxDxStages;  // [NS] Wt block read by the MMA
  uint64_t* done = wt_empty + kMaxDxStages;     // every MMA of the CTA finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int w = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 5);   // MMA commit + the 4 warps of one densify set
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
      const uint32_t bytes = (uint32_t)(BH + kK) * RB;  // dY tile + weight block
      const bool group_major = a.dy_gstride != kG;
      // a ring load from HBM takes longer than the ring's MMA work: the tiles of
      // later groups are requested into L2 ahead of their ring loads
      auto prefetch = [&](int64_t g) {
        if (group_major) prefetch_l2(a.dY + g * a.dy_gstride + (int64_t)256 * bh * kG, (uint32_t)(BH * RB));
        prefetch_l2(a.W + g * kG * kK, (uint32_t)(kG * kK * 2));
        prefetch_l2(a.idx + g * kK, (uint32_t)(kK * 4));
      };
      for (int i = 0; i < kDxPrefetch && i < n; ++i) prefetch(g0 + i);
      int st = 0, ph = 0, issued = 0;
      for (int i = 0; i < n; ++i) {
        const int64_t g = g0 + i;
        if (i + kDxPrefetch < n) prefetch(g + kDxPrefetch);
        if (!wait_or_abort(&empty[st], ph ^ 1, abort_flag)) break;
        ++issued;
        mbar_arrive_expect_tx(&full[st], bytes);
        tma_load_2d(DYS(st), &tm_dy, (int)(g * a.dy_xg), (int)(g * a.dy_yg + 256 * bh), &full[st]);
#pragma unroll
        for (int blk = 0; blk < kK / 64; ++blk)
          tma_load_2d(WS(st) + (uint32_t)(blk * kG * 128), &tm_w, 64 * blk, (int)(g * kG), &full[st]);
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
    const uint32_t idesc = make_idesc(1, 0, 0, 128, (uint32_t)NB);
    int st = 0, ph = 0;
    for (int i = 0; i < n; ++i) {
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[st], ph, abort_flag))) break;
      if (!__all_sync(0xffffffffu, wait_or_abort(&wt_full[st], ph, abort_flag))) break;
      tc_fence_after();
      if (lane == 0) {
        for (int t = 0; t < MT; ++t)
#pragma unroll
          for (int kk = 0; kk < kG / 16; ++kk) {
            const uint64_t ad =
                make_sdesc(DYS(st) + (uint32_t)(t * 128 * RB + kk * 32), 16, 8 * RB, layout_for_rows(RB));
            const uint64_t bd = make_sdesc(WT(st) + (uint32_t)(kk * 32), 16, 8 * RB, layout_for_rows(RB));
            mma_ss<false>(tmem + (uint32_t)(t * 256), ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
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
    const int set = (w - 2) >> 2;          // groups i = set, set + 2, ...
    const int s = (threadIdx.x - 64) & 127;  // this thread's slot
    const bool slot_ok = s < kK;
    // column s of a weight block: 64-slot block s/64, 16-byte chunk (s%64)/8 of each
    // 128-byte row (TMA 128-byte swizzle), element s%8
    const uint32_t wcol = (uint32_t)((s >> 6) * kG * 128 + (s & 7) * 2);
    const uint32_t wchunk = (uint32_t)((s & 63) >> 3);
    // the slot's feature in group i of the chunk (-1: no such group or slot)
    auto feat = [&](int i) -> int { return slot_ok && i >= 0 && i < n ? a.idx[(g0 + i) * kK + s] : -1; };
    // features of this set's next three groups, and of the groups NS before them
    // (the previous users of the same ring stages), loaded ahead
    int fa = feat(set), fb = feat(set + 2), fc = feat(set + 4);
    int oa = feat(set - NS), ob = feat(set + 2 - NS), oc = feat(set + 4 - NS);
    // ring position of group i, advanced by two groups per iteration (NS >= 2)
    int st = set;
    uint32_t ph = 0;
    for (int i = set; i < n; i += 2) {
      const int f = fa - f0, r = oa - f0;
      const bool act = fa >= 0 && f >= 0 && f < nf;
      const bool old = oa >= 0 && r >= 0 && r < nf;
      fa = fb;
      fb = fc;
      fc = feat(i + 6);
      oa = ob;
      ob = oc;
      oc = feat(i + 6 - NS);
      uint8_t* wt = gbase + Lo.wt + st * Lo.wt_stride;
      // the MMA of group i - NS has read this stage's Wt block: clear its rows
      const bool ok = __all_sync(0xffffffffu, wait_or_abort(&wt_empty[st], ph ^ 1u, abort_flag));
      if (ok) {
        if (old) {
#pragma unroll
          for (int cc = 0; cc < kG / 8; ++cc)
            *reinterpret_cast<uint4*>(wt + swz_rows((uint32_t)(r * RB + cc * 16), RB)) = make_uint4(0, 0, 0, 0);
        }
      }
      // every old row is clear before any new row is written (two slots of
      // different groups may share a feature)
      named_bar(1 + set, 128);
      const bool ok2 = ok && __all_sync(0xffffffffu, wait_or_abort(&full[st], ph, abort_flag));
      if (ok2) {
        if (act) {
          const uint8_t* col = gbase + Lo.w + st * Lo.w_stride + wcol;
          uint32_t pk[kG / 2];
#pragma unroll
          for (int l = 0; l < kG; l += 2) {
            const uint32_t lo = *reinterpret_cast<const uint16_t*>(col + l * 128 + ((wchunk ^ (l & 7)) << 4));
            const uint32_t hi =
                *reinterpret_cast<const uint16_t*>(col + (l + 1) * 128 + ((wchunk ^ ((l + 1) & 7)) << 4));
            pk[l / 2] = lo | (hi << 16);
          }
#pragma unroll
          for (int cc = 0; cc < kG / 8; ++cc)
            *reinterpret_cast<uint4*>(wt + swz_rows((uint32_t)(f * RB + cc * 16), RB)) =
                make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0 && ok2) {
        mbar_arrive(&empty[st]);
        mbar_arrive(&wt_full[st]);
      }
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

size_t dx_smem(int Bp, int band, int k, int G, int ns) { return v2::dx_layout(Bp, band, k, G, ns).total; }

// Feature bands and ring depth of the dX pass: bands of at most 256 features
// (the widest MMA N), as few as cover d, split evenly in multiples of 16; the
// deepest ring (up to six stages) that fits in the shared memory left after
// `reserve` bytes.  Returns false when two stages do not fit.
bool dx_supported(int G, int k, int Bp) {
  return (G == 16 || G == 32 || G == 64) && (k == 64 || k == 128) && Bp <= 512;
}

bool dx_config(int G, int k, int d, int Bp, size_t smem_optin, size_t reserve, int* band, int* n_bands, int* ns) {
  Bp = Bp < 256 ? Bp : 256;  // a CTA covers a batch half of up to 256 rows
  const int nb = (d + 255) / 256;
  const int bw = (((d + nb - 1) / nb) + 15) & ~15;
  int best = 0;
  for (int st = 2; st <= v2::kMaxDxStages; ++st)
    if (dx_smem(Bp, bw, k, G, st) + reserve <= smem_optin) best = st;
  if (!best) return false;
  *band = bw;
  *n_bands = nb;
  *ns = best;
  return true;
}

// dY of the dX pass, either the group-major buffer [n_groups, Bp, G] of the fused
// step (dy_gstride = Bp*G, dy_rstride = G; rows past B hold zeros) or a caller's
// row-major [B, L] (dy_gstride = G, dy_rstride = L; rows past B are outside the
// tensor and read as zeros).
template <int kG, int kK>
cudaError_t launch_dx_t(v2::DxArgs a, const void* dY, const void* W, cudaStream_t st) {
  const int BH = a.sh.Bp < 256 ? a.sh.Bp : 256;
  const size_t smem = dx_smem(BH, a.band, kK, kG, a.ns);
  auto kern = v2::k_dx_band<kG, kK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_dy, tm_w;
  const bool group_major = a.dy_gstride != kG;  // row-major [B, L] has dy_gstride = G
  if (group_major) {
    e = tmap_2d(&tm_dy, dY, kG, (uint64_t)a.sh.n_groups * a.sh.Bp, (uint64_t)kG * 2, kG, (uint32_t)BH);
    a.dy_xg = 0;
    a.dy_yg = a.sh.Bp;
  } else {
    e = tmap_2d(&tm_dy, dY, (uint64_t)a.sh.L, (uint64_t)a.sh.B, (uint64_t)a.dy_rstride * 2, kG, (uint32_t)BH);
    a.dy_xg = kG;
    a.dy_yg = 0;
  }
  if (e == cudaSuccess) e = tmap_2d(&tm_w, W, kK, (uint64_t)a.sh.L, (uint64_t)kK * 2, 64, kG);
  if (e != cudaSuccess) return e;
  const int grid = a.n_bands * a.n_halves * a.n_chunks;
  kern<<<grid, v2::kDxThreads, smem, st>>>(a, tm_dy, tm_w);
  return cudaGetLastError();
}

cudaError_t launch_dx(int G, int k, const v2::DxArgs& a, const void* dY, const void* W, cudaStream_t st) {
  HASTE_V2_DISPATCH(launch_dx_t, a, dY, W, st)
}

}  // namespace tail2
}  // namespace haste
