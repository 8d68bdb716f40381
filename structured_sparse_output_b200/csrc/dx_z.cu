// dx_z.cu -- dX of the group-shared sparse tail (HASTE, "Hardware-Aware Dynamic
// Sparse Training for Large Output Spaces", Methodology 1: the G labels of group g
// read the k features I_g, so the group's share of the input gradient,
// Z_g = dY_g . W_g [B x k], lands in the columns I_g of dX).
//
// k_dx_z -- one CTA per (group chunk c, 128-row batch tile t, feature part p):
//   warp 0 (one thread)  producer: per group, the dY tile (128 rows x G labels),
//                        the G x k weight block and the group's index row into a
//                        ring stage (TMA tiles and one bulk copy);
//   warp 1 (one thread)  MMA: Z = dY_g[tile] . W_g[:, 64-slot block], M = 128 batch
//                        rows, N = 64 slots, K = G, into a 2-deep TMEM ring, for
//                        the blocks that hold a feature of part p (an index row
//                        is sorted, so a part's slots are one contiguous run and
//                        most groups need only some of the blocks);
//   warps 2-9            scatter: thread = batch row.  Column s of Z is added to
//                        the accumulator column of feature idx[g, s] (TMEM, fp32,
//                        one column per feature of the part).  Every column
//                        receives its (group, slot) terms in ascending group
//                        order -- the order of the feature's inverse-map segment
//                        -- from one thread, with no atomics.  At the end the
//                        accumulator is written out as the chunk's partial.
// k_dx_reduce (tail.cu) sums the chunk partials in chunk order.
//
// TMEM: columns [0, 128) hold the Z ring, [128, 128 + part width) the
// accumulator; the part width is at most 384, so a CTA allocates all 512 columns
// and runs alone on its SM.

#include "tail.cuh"

namespace haste {
namespace v2 {

struct DxzArgs {
  TailShape sh;
  const int32_t* idx;
  const __nv_bfloat16* dY;  // for L2 prefetches
  const __nv_bfloat16* W;
  float* dX_part;  // [n_chunks, d, Bp]
  int n_chunks, n_parts, part_w, ns;
  int dy_group_major;  // 1: the fused step's buffer [n_groups, Bp, G]; 0: the caller's [B, L]
};

constexpr int kDxzMaxStages = 8;
constexpr int kDxzThreads = 320;  // producer warp, MMA warp, 8 scatter warps
constexpr int kDxzPrefetch = 8;   // groups ahead of the ring loads requested into L2
constexpr int kDxzAccCol = 128;   // first accumulator column (after the Z ring)
constexpr int kDxzMaxPart = 384;  // features per part: 128 + 384 = 512 TMEM columns
constexpr size_t kDxzMinSmem = 120 * 1024;  // keeps one CTA per SM (it takes all of TMEM)

struct DxzLayout {
  uint32_t dy_stride, w_stride, ix_stride, dy, w, ix, bars, total;
};
// ns stages of (dY tile [128][G], weight block [k/64][G][64], index row [k]).
__host__ __device__ inline DxzLayout dxz_layout(int k, int G, int ns) {
  DxzLayout L;
  L.dy_stride = (uint32_t)((128 * G * 2 + 1023) & ~1023);
  L.w_stride = (uint32_t)(((k / 64) * G * 128 + 1023) & ~1023);
  L.ix_stride = (uint32_t)(k * 4);
  uint32_t off = 0;
  L.dy = off;
  off += ns * L.dy_stride;
  L.w = off;
  off += ns * L.w_stride;
  L.ix = off;
  off += ns * L.ix_stride;
  L.bars = off;
  off += 256;
  L.total = off + 1024;
  return L;
}

__device__ __forceinline__ void tmem_ld16u(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <int kG, int kK>
__global__ void __launch_bounds__(kDxzThreads, 1)
    k_dx_z(DxzArgs a, const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int RB = kG * 2;       // bytes of a dY row (K-major A operand)
  constexpr int NBLK = kK / 64;    // 64-slot blocks of a weight block
  const int NS = a.ns;
  const TailShape sh = a.sh;
  const int n_bt = sh.Bp / 128;
  const int per_chunk = n_bt * a.n_parts;
  const int c = blockIdx.x / per_chunk;
  const int t = (blockIdx.x % per_chunk) / a.n_parts;
  const int p = blockIdx.x % a.n_parts;
  const int f0 = p * a.part_w;
  const int nf = min(sh.d, f0 + a.part_w) - f0;  // features of this part
  const int64_t g0 = (int64_t)c * sh.n_groups / a.n_chunks;
  const int64_t g1 = (int64_t)(c + 1) * sh.n_groups / a.n_chunks;
  const int n = (int)(g1 - g0);

  const DxzLayout Lo = dxz_layout(kK, kG, NS);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  auto DYS = [&](int st) -> uint32_t { return base + Lo.dy + st * Lo.dy_stride; };
  auto WS = [&](int st) -> uint32_t { return base + Lo.w + st * Lo.w_stride; };
  auto IXS = [&](int st) -> const int32_t* {
    return reinterpret_cast<const int32_t*>(gbase + Lo.ix + st * Lo.ix_stride);
  };
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;                      // [NS] stage landed (1 + tx bytes)
  uint64_t* empty = full + kDxzMaxStages;     // [NS] stage read: MMA commit + 8 scatter warps
  uint64_t* zfull = empty + kDxzMaxStages;    // [2] Z block in TMEM
  uint64_t* zfree = zfull + 2;                // [2] Z block read (8 scatter warps)
  uint64_t* done = zfree + 2;                 // every MMA of the CTA finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 9);
    }
    for (int z = 0; z < 2; ++z) {
      mbar_init(&zfull[z], 1);
      mbar_init(&zfree[z], 8);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (w == 1) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  // Block j (slots [64j, 64j+64)) of a group holds a feature of this part; both
  // the MMA warp and the scatter warps decide this from the staged index row.
  auto need = [&](const int32_t* ix, int j) -> bool { return ix[64 * j + 63] >= f0 && ix[64 * j] < f0 + nf; };

  if (w == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t bytes = (uint32_t)(128 * RB + kK * RB + kK * 4);  // dY tile + weight block + index row
      // ring loads from HBM take longer than a group's work: later groups' tiles
      // are requested into L2 first (the weight block and indices by part 0 only)
      auto prefetch = [&](int64_t g) {
        if (a.dy_group_major) prefetch_l2(a.dY + (g * sh.Bp + t * 128) * kG, (uint32_t)(128 * RB));
        if (p == 0) {
          prefetch_l2(a.W + g * kG * kK, (uint32_t)(kG * kK * 2));
          prefetch_l2(a.idx + g * kK, (uint32_t)(kK * 4));
        }
      };
      for (int i = 0; i < kDxzPrefetch && i < n; ++i) prefetch(g0 + i);
      int st = 0, ph = 0, issued = 0;
      for (int i = 0; i < n; ++i) {
        const int64_t g = g0 + i;
        if (i + kDxzPrefetch < n) prefetch(g + kDxzPrefetch);
        if (!wait_or_abort(&empty[st], ph ^ 1, abort_flag)) break;
        ++issued;
        mbar_arrive_expect_tx(&full[st], bytes);
        if (a.dy_group_major)
          tma_load_2d(DYS(st), &tm_dy, 0, (int)(g * sh.Bp + t * 128), &full[st]);
        else
          tma_load_2d(DYS(st), &tm_dy, (int)(g * kG), t * 128, &full[st]);
#pragma unroll
        for (int blk = 0; blk < NBLK; ++blk)
          tma_load_2d(WS(st) + (uint32_t)(blk * kG * 128), &tm_w, 64 * blk, (int)(g * kG), &full[st]);
        bulk_load(base + Lo.ix + st * Lo.ix_stride, a.idx + g * kK, (uint32_t)(kK * 4), &full[st]);
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
    // ----------------------------------------------------------------- MMA
    const uint32_t idesc = make_idesc(1, 0, 1, 128, 64);  // A K-major (dY), B MN-major (W, slots contiguous)
    int st = 0, ph = 0, zb = 0, zph = 0;
    bool ok = true;
    for (int i = 0; ok && i < n; ++i) {
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[st], ph, abort_flag))) break;
      const int32_t* ix = IXS(st);
      for (int j = 0; j < NBLK; ++j) {
        if (!need(ix, j)) continue;
        if (!__all_sync(0xffffffffu, wait_or_abort(&zfree[zb], zph ^ 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < kG / 16; ++kk) {
            const uint64_t ad = make_sdesc(DYS(st) + (uint32_t)(kk * 32), 16, 8 * RB, layout_for_rows(RB));
            const uint64_t bd =
                make_sdesc(WS(st) + (uint32_t)(j * kG * 128 + kk * 16 * 128), kG * 128, 1024, kLayoutSw128);
            mma_ss<false>(tmem + (uint32_t)(zb * 64), ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&zfull[zb]);
        }
        __syncwarp();
        if (++zb == 2) {
          zb = 0;
          zph ^= 1;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(&empty[st]);
      __syncwarp();
      if (++st == NS) {
        st = 0;
        ph ^= 1;
      }
    }
    // also after an abort: TMEM is freed only once every issued MMA has finished
    if (lane == 0) mma_commit(done);
    __syncwarp();
    (void)__all_sync(0xffffffffu, mbar_wait(done, 0));
  } else {
    // ------------------------------------------------------------- scatter
    // warp (q, h): TMEM lane quarter q (batch rows 32q.. of the tile), the 16-slot
    // chunks h and h + 2 of each block.  Every warp runs one iteration per group
    // and meets the others at a named barrier after it (a feature can sit in
    // different chunks of consecutive groups, so the warps of a quarter must not
    // overlap groups); after an abort the iterations skip their work.
    const int q = w & 3, h = (w - 2) >> 2;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t acc = tmem + lane_off + kDxzAccCol;
    for (int col = 16 * h; col < kDxzMaxPart; col += 32) tmem_st16_zero(acc + (uint32_t)col);
    tmem_wait_st();
    tc_fence_before();
    named_bar(1, 256);
    tc_fence_after();
    const uint32_t unf = (uint32_t)nf;
    int st = 0, ph = 0, zb = 0, zph = 0;
    for (int i = 0; i < n; ++i) {
      const bool okf = __all_sync(0xffffffffu, wait_or_abort(&full[st], ph, abort_flag));
      if (okf) {
        const int32_t* ix = IXS(st);
        for (int j = 0; j < NBLK; ++j) {
          if (!need(ix, j)) continue;
          if (!__all_sync(0xffffffffu, wait_or_abort(&zfull[zb], zph, abort_flag))) break;
          tc_fence_after();
#pragma unroll 1
          for (int cc = h; cc < 4; cc += 2) {
            const int s0 = 64 * j + 16 * cc;
            if (ix[s0 + 15] < f0 || ix[s0] >= f0 + nf) continue;  // no feature of the part in this chunk
            uint32_t z[16], v[16];
            int fe[16];
            tmem_ld16u(tmem + lane_off + (uint32_t)(zb * 64 + 16 * cc), z);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              fe[e] = ix[s0 + e] - f0;
              v[e] = (uint32_t)fe[e] < unf ? tmem_ld1(acc + (uint32_t)fe[e]) : 0u;
            }
            tmem_wait_ld16(z);
            tmem_wait_ld16(v);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if ((uint32_t)fe[e] < unf)
                tmem_st1(acc + (uint32_t)fe[e], __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(z[e])));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&zfree[zb]);
          if (++zb == 2) {
            zb = 0;
            zph ^= 1;
          }
        }
      }
      // this group's accumulator updates are complete before any warp starts the next
      tmem_wait_st();
      tc_fence_before();
      named_bar(1, 256);
      tc_fence_after();
      if (lane == 0 && okf) mbar_arrive(&empty[st]);
      if (++st == NS) {
        st = 0;
        ph ^= 1;
      }
    }
    // ------------------------------------------------------------ epilogue
    const bool fin = __all_sync(0xffffffffu, mbar_wait(done, 0)) && !*abort_flag;
    tc_fence_after();
    if (fin) {
      const int b = t * 128 + q * 32 + lane;
      for (int col = 16 * h; col < nf; col += 32) {
        float v[16];
        tmem_ld16(acc + (uint32_t)col, v);
        tmem_wait_ld();
        float* dst = a.dX_part + ((int64_t)c * sh.d + f0 + col) * sh.Bp + b;
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (col + e < nf) dst[(int64_t)e * sh.Bp] = v[e];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace v2

// ------------------------------------------------------------- host side
namespace tail2 {

bool dxz_supported(int G, int k, int Bp) {
  return (G == 16 || G == 32 || G == 64) && (k == 64 || k == 128) && Bp <= 512;
}

size_t dxz_smem(int k, int G, int ns) {
  return std::max(v2::dxz_layout(k, G, ns).total, (uint32_t)v2::kDxzMinSmem);
}

// Feature parts of the dX pass (as few as keep a part within 384 features, split
// evenly) and the deepest ring (up to eight stages) that fits in the shared
// memory left after `reserve` bytes.  Returns false when two stages do not fit.
bool dxz_config(int G, int k, int d, size_t smem_optin, size_t reserve, int* n_parts, int* part_w, int* ns) {
  const int np = (d + v2::kDxzMaxPart - 1) / v2::kDxzMaxPart;
  int best = 0;
  for (int st = 2; st <= v2::kDxzMaxStages; ++st)
    if (dxz_smem(k, G, st) + reserve <= smem_optin) best = st;
  if (!best) return false;
  *n_parts = np;
  *part_w = (d + np - 1) / np;
  *ns = best;
  return true;
}

template <int kG, int kK>
cudaError_t launch_dxz_t(v2::DxzArgs a, const void* dY, const void* W, cudaStream_t st) {
  const size_t smem = dxz_smem(kK, kG, a.ns);
  auto kern = v2::k_dx_z<kG, kK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_dy, tm_w;
  if (a.dy_group_major)
    e = tmap_2d(&tm_dy, dY, kG, (uint64_t)a.sh.n_groups * a.sh.Bp, (uint64_t)kG * 2, kG, 128);
  else
    e = tmap_2d(&tm_dy, dY, (uint64_t)a.sh.L, (uint64_t)a.sh.B, (uint64_t)a.sh.L * 2, kG, 128);
  if (e == cudaSuccess) e = tmap_2d(&tm_w, W, kK, (uint64_t)a.sh.L, (uint64_t)kK * 2, 64, kG);
  if (e != cudaSuccess) return e;
  const int grid = a.n_chunks * (a.sh.Bp / 128) * a.n_parts;
  kern<<<grid, v2::kDxzThreads, smem, st>>>(a, tm_dy, tm_w);
  return cudaGetLastError();
}

cudaError_t launch_dxz(int G, int k, const v2::DxzArgs& a, const void* dY, const void* W, cudaStream_t st) {
  HASTE_V2_DISPATCH(launch_dxz_t, a, dY, W, st)
}

}  // namespace tail2
}  // namespace haste
