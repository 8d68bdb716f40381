// tail_v2.cu -- warp-specialised, pipelined bf16 kernels of the group-shared sparse
// tail (HASTE, "Hardware-Aware Dynamic Sparse Training for Large Output Spaces",
// Methodology 1: labels in groups of G share one fan-in set I_g of k features).
//
// k_step2 -- fused forward + BCE gradient + dW, one group per iteration:
//   warps 0-3  producers: the gather-once tile X[:, I_g] (k rows of X^T) and the
//              G x k weight block, staged with cp.async into a 2-stage ring; warps
//              0 and 2 fill stage 0, warps 1 and 3 stage 1;
//   warp 4     MMA issuer (one thread): issues each group's forward and dW
//              product as soon as its inputs are ready, so the tensor core works
//              while the epilogue runs;
//   warps 5-12 epilogue: logits leave TMEM only as the BCE gradient (bf16, into
//              shared memory: the dW operand, and the tile that the MMA thread
//              writes to the gradient buffer of the dX pass with one TMA store,
//              items of 64 / G groups side by side in 128-byte rows); the BCE of group i+1 comes before the dW readout of
//              group i, so the dW product runs behind it.  The readout
//              writes dW, or (kUpd > 0) applies an SGD update to the group's
//              weights while dW is on chip: M' = momentum * M + dW (kUpd = 2) or
//              M' = dW (kUpd = 1), W' = W - lr * M', with W' written to a
//              separate buffer (the dX pass still reads W) and M' over M.
//
// The dX pass that reads the gradient buffer is in dx_band.cu.

#include "tail.cuh"

namespace haste {
namespace v2 {

struct StepArgs {
  TailShape sh;
  const int32_t* idx;
  __nv_bfloat16* dW;      // kUpd = 0
  __nv_bfloat16* W_out;   // kUpd > 0: updated weights [L, k]
  __nv_bfloat16* M;       // kUpd = 2: momentum [L, k], updated in place
  float lr, momentum;
  __nv_bfloat16* dY_out;  // gradient buffer [n_groups / (64 / G)][Bp][64] of the dX pass
  float* loss_part;
  const int32_t* pos_ptr;
  const int32_t* pos_ids;
  float grad_scale;
};

// ------------------------------------------------------------ smem layouts
struct StepLayout {
  uint32_t xg[2], wg[2], dy[2], bars, total;
};
__host__ __device__ inline StepLayout step_layout(int Bp, int k, int G) {
  StepLayout L;
  const uint32_t xg = (uint32_t)((Bp / 64) * k * 128 + (k < 128 ? (128 - k) * 128 : 0));
  const uint32_t wg = (uint32_t)((k / 64) * G * 128);
  const uint32_t dy = (uint32_t)(Bp * G * 2);
  uint32_t off = 0;
  for (int s = 0; s < 2; ++s) { L.xg[s] = off; off += xg; }
  for (int s = 0; s < 2; ++s) { L.wg[s] = off; off += wg; }
  for (int s = 0; s < 2; ++s) { L.dy[s] = off; off += (dy + 1023u) & ~1023u; }
  L.bars = off;
  off += 256;
  L.total = off + 1024;
  return L;
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Bounded wait; on timeout the CTA-wide abort flag is raised.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity, g_wait_limit_ns)) {
    *abort_flag = 1;
    return false;
  }
  return true;
}

// A producer thread publishes its finished copies to the tensor core (proxy
// fence) before arriving on the stage's full barrier.
__device__ __forceinline__ void publish_all(uint64_t* full_bar) {
  cp_async_wait_all();
  fence_proxy_async_smem();
  mbar_arrive(full_bar);
}

// ============================================================ k_step2
constexpr int kStepProd = 4;       // producer warps: two per ring stage
constexpr int kStepMma = kStepProd;  // warp id of the MMA issuer
constexpr int kStepEpi = 8;        // epilogue warps: 4 lane quarters x 2 column halves
constexpr int kStepThreads = 32 * (kStepProd + 1 + kStepEpi);  // producers, MMA warp, epilogue warps
constexpr int kMaxPosReg = 8;      // positives per batch row kept in registers

template <int kG, int kK, int kUpd>
__global__ void __launch_bounds__(kStepThreads, 1)
    k_step2(StepArgs a, const __nv_bfloat16* __restrict__ Xt, const __nv_bfloat16* __restrict__ W,
            const __grid_constant__ CUtensorMap tm_dy) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int RB = kG * 2;   // bytes of one dY row in shared memory
  constexpr int CH = kG / 2;   // label columns per epilogue half
  constexpr int kRowsPerThr = kK / 4;
  const TailShape sh = a.sh;
  const int Bp = sh.Bp, n_bt = Bp / 128;
  const StepLayout Lo = step_layout(Bp, kK, kG);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;             // [2] stage loaded (count: one producer half)
  uint64_t* empty = bars + 2;        // [2] stage free
  uint64_t* fwd_full = bars + 4;     // [2] logits in TMEM
  uint64_t* dy_full = bars + 6;      // [2] dY in shared memory
  uint64_t* dw_full = bars + 8;      // [2] dW in TMEM
  uint64_t* tmem_empty = bars + 10;  // [2] dW accumulator D read out
  uint64_t* done = bars + 12;        // every MMA of the CTA finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  float* red = reinterpret_cast<float*>(tslot + 2);  // kStepEpi warp partials

  const int w = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 32 * kStepProd / 2);
      mbar_init(&empty[s], 1);
      mbar_init(&fwd_full[s], 1);
      mbar_init(&dy_full[s], kStepEpi);
      mbar_init(&dw_full[s], 1);
      mbar_init(&tmem_empty[s], kStepEpi);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // TMEM: forward accumulators F[2] (n_bt*G columns each), dW accumulators D[2]
  const uint32_t f_cols = (uint32_t)(n_bt * kG);
  const uint32_t ncols = tmem_cols_for(2 * f_cols + 2 * kG);
  if (w == kStepMma) {
    tmem_alloc(tslot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  auto F = [&](int s) -> uint32_t { return tmem + (s ? f_cols : 0u); };
  auto D = [&](int s) -> uint32_t { return tmem + 2 * f_cols + (s ? (uint32_t)kG : 0u); };
  auto XG = [&](int s) -> uint32_t { return base + (s ? Lo.xg[1] : Lo.xg[0]); };
  auto WG = [&](int s) -> uint32_t { return base + (s ? Lo.wg[1] : Lo.wg[0]); };
  auto DY = [&](int s) -> uint32_t { return s ? Lo.dy[1] : Lo.dy[0]; };

  // contiguous chunk of groups per CTA
  const int64_t gb = (int64_t)blockIdx.x * sh.n_groups / gridDim.x;
  const int64_t ge = (int64_t)(blockIdx.x + 1) * sh.n_groups / gridDim.x;
  const int n_items = (int)(ge - gb);

  if (w < kStepProd) {
    // ------------------------------------------------- cp.async producers
    // warps (half, part) fill stage half with the items i = half, half+2, ...;
    // each of the two warps of a stage copies every other group of four rows.
    // Lane (rg, sub) copies the 16-byte chunk sub of every 128-byte segment of
    // its rows, so that 8 consecutive lanes read one segment; the feature
    // indices of its rows sit in registers.
    constexpr int P = kStepProd / 2;
    constexpr int kRows = kRowsPerThr / P;
    const int half = w & 1, part = w >> 1, ht = lane;
    const int sub = ht & 7, rg = ht >> 3;
    const uint32_t xg = XG(half), wg = WG(half);
    int i = half;
    for (; i < n_items; i += 2) {
      const int64_t g = gb + i;
      // this half's next group: weight block and indices into L2 (from HBM they
      // would stretch the gather of that group)
      if (part == 0 && lane == 0 && i + 2 < n_items) {
        prefetch_l2(W + (g + 2) * kG * kK, (uint32_t)(kG * kK * 2));
        prefetch_l2(a.idx + (g + 2) * kK, (uint32_t)(kK * 4));
        if constexpr (kUpd == 2) prefetch_l2(a.M + (g + 2) * kG * kK, (uint32_t)(kG * kK * 2));  // read by the update
      }
      // the index loads are in flight while this half waits for its stage
      int idx_cur[kRows];
#pragma unroll
      for (int m = 0; m < kRows; ++m) idx_cur[m] = a.idx[g * kK + rg + 4 * (m * P + part)];
      if (!wait_or_abort(&empty[half], ((i >> 1) & 1) ^ 1, abort_flag)) break;
      const int nbb = Bp / 64;
#pragma unroll
      for (int m = 0; m < kRows; ++m) {
        const int sl = rg + 4 * (m * P + part);
        const __nv_bfloat16* src = Xt + (int64_t)idx_cur[m] * Bp + sub * 8;
        const uint32_t dst = xg + sw128((uint32_t)(sl * 128 + sub * 16));  // swizzle is the same in every block
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
          if (bb < nbb) cp_async16(dst + (uint32_t)(bb * kK * 128), src + bb * 64, 16);
      }
      // weight block of the group (contiguous G x k), chunks split between the warps
      const __nv_bfloat16* wsrc = W + g * (int64_t)kG * kK;
      constexpr int cpr = kK / 8;
#pragma unroll 4
      for (int c0 = 32 * part; c0 < kG * cpr; c0 += 32 * P) {
        const int c = c0 + ht;
        const int j = c / cpr, cc = c % cpr;
        cp_async16(wg + sw128((uint32_t)((cc >> 3) * kG * 128 + j * 128 + (cc & 7) * 16)),
                   wsrc + (int64_t)j * kK + cc * 8, 16);
      }
      cp_async_commit();
      publish_all(&full[half]);
    }
    cp_async_wait_all();
  } else if (w == kStepMma) {
    // ------------------------------------------------------------ MMA issuer
    // Forwards and dW products are issued as their inputs become ready, not in a
    // fixed interleave: fwd(j) needs its gathered stage (full) and F(j&1) free,
    // which holds once dW(j-2) was issued (its BCE had finished reading F);
    // dW(j) needs the BCE of j (dy_full) and D(j&1) read out for j-2
    // (tmem_empty).  Lane 0 polls; the decisions are broadcast so the warp stays
    // converged.  No progress for the wait limit raises the abort flag.
    const uint32_t idesc_f = make_idesc(1, 1, 0, 128, kG);
    const uint32_t idesc_w = make_idesc(1, 0, 1, 128, kG);
    int nf = 0, nd = 0;
    uint64_t t_last = globaltimer_ns();
    const uint64_t limit = g_wait_limit_ns;
    while (nd < n_items) {
      if (*abort_flag) break;
      bool did = false;
      if (nf < n_items && nf <= nd + 1) {
        const int s = nf & 1;
        const bool rdy = __shfl_sync(0xffffffffu, lane == 0 ? mbar_try_wait(&full[s], (nf >> 1) & 1) : false, 0);
        if (rdy) {
          if (lane == 0) {
            tc_fence_after();
            for (int t = 0; t < n_bt; ++t)
              for (int kk = 0; kk < kK / 16; ++kk) {
                const uint64_t ad = make_sdesc(XG(s) + (uint32_t)(t * 2 * kK * 128 + kk * 16 * 128),
                                               (uint32_t)kK * 128, 1024, kLayoutSw128);
                const uint64_t bd =
                    make_sdesc(WG(s) + (uint32_t)((kk / 4) * kG * 128 + (kk % 4) * 32), 16, 1024, kLayoutSw128);
                mma_ss<false>(F(s) + (uint32_t)(t * kG), ad, bd, idesc_f, kk > 0 ? 1u : 0u);
              }
            // the BCE of this group rewrites the dY tile of group nf - 2, whose
            // store may be the latest one issued: every store must have read its
            // tile before the BCE is released (the forward's MMAs run meanwhile)
            bulk_wait_read<0>();
            mma_commit(&fwd_full[s]);
          }
          __syncwarp();
          ++nf;
          did = true;
        }
      }
      if (nd < nf) {
        const int s = nd & 1;
        const bool rdy = __shfl_sync(0xffffffffu,
                                     lane == 0 ? (mbar_try_wait(&dy_full[s], (nd >> 1) & 1) &&
                                                  mbar_try_wait(&tmem_empty[s], ((nd >> 1) & 1) ^ 1))
                                               : false,
                                     0);
        if (rdy) {
          if (lane == 0) {
            tc_fence_after();
            for (int kk = 0; kk < Bp / 16; ++kk) {
              const int b = kk * 16;
              const uint64_t ad =
                  make_sdesc(XG(s) + (uint32_t)((b / 64) * kK * 128 + (kk % 4) * 32), 16, 1024, kLayoutSw128);
              const uint64_t bd = make_sdesc(base + DY(s) + (uint32_t)(b * RB), 16, 8 * RB, layout_for_rows(RB));
              mma_ss<false>(D(s), ad, bd, idesc_w, kk > 0 ? 1u : 0u);
            }
            mma_commit(&dw_full[s]);
            mma_commit(&empty[s]);
            // the group's gradient tile to the dX pass's buffer: columns of its
            // item (64 / G consecutive groups, 64 labels), the item's Bp rows
            {
              const int64_t g = gb + nd;
              constexpr int NG = 64 / kG;
              tma_store_2d(&tm_dy, base + DY(s), (int)(g % NG) * kG, (int)((g / NG) * Bp));
            }
            bulk_commit();
          }
          __syncwarp();
          ++nd;
          did = true;
        }
      }
      if (did) {
        t_last = globaltimer_ns();
      } else {
        if (globaltimer_ns() - t_last > limit) {
          if (lane == 0) {
            *abort_flag = 1;
            record_error(kErrTimeout);
          }
          __syncwarp();
          break;
        }
        __nanosleep(32);
      }
    }
    // Also after an abort: the CTA frees TMEM and exits only once every MMA it
    // issued has finished writing TMEM and reading shared memory, and its stores
    // are complete.
    if (lane == 0) {
      mma_commit(done);
      bulk_wait_all();
    }
    __syncwarp();
    (void)__all_sync(0xffffffffu, mbar_wait(done, 0));
  } else {
    // ------------------------------------------------------------- epilogue
    // warp (q, hh): TMEM lane quarter q, label columns [hh*CH, hh*CH + CH)
    const int ew = w - kStepMma - 1, q = w & 3, hh = ew >> 2;
    const int r = q * 32 + lane;  // row inside a 128-row tile (and dW slot)
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float scale = a.grad_scale;
    float loss_acc = 0.f;
    // this thread's positives (tail-local ids), one batch row per 128-row tile
    int pos[2][kMaxPosReg];
    int npos[2] = {0, 0}, pbeg[2] = {0, 0};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int b = t * 128 + r;
      if (t < n_bt && b < sh.B) {
        pbeg[t] = a.pos_ptr[b];
        npos[t] = a.pos_ptr[b + 1] - pbeg[t];
      }
#pragma unroll
      for (int e = 0; e < kMaxPosReg; ++e) pos[t][e] = e < npos[t] ? a.pos_ids[pbeg[t] + e] : -1;
    }
    auto bce = [&](int i) -> bool {
      const int64_t g = gb + i;
      const int s = i & 1;
      if (!wait_or_abort(&fwd_full[s], (i >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const int64_t l0 = g * kG + hh * CH;  // first label of this warp's columns
      uint8_t* dyrow = gbase + DY(s);
      // every logit of this thread's columns in both batch tiles is requested from
      // TMEM before the first is used: one load latency per group, not one per chunk
      constexpr int NC = CH < 16 ? CH : 16;
      float zall[2][CH];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t < n_bt) {
#pragma unroll
          for (int c = 0; c < CH; c += 16) {
            if constexpr (NC == 8) tmem_ld8(F(s) + lane_off + (uint32_t)(t * kG + hh * CH + c), &zall[t][c]);
            else tmem_ld16(F(s) + lane_off + (uint32_t)(t * kG + hh * CH + c), *reinterpret_cast<float(*)[16]>(&zall[t][c]));
          }
        }
      }
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= n_bt) break;
        const int b = t * 128 + r;
        const bool live = b < sh.B;
        const float sl = live ? scale : 0.f, hs = 0.5f * sl;  // rows beyond B get dY = 0
        uint32_t ym = 0;
#pragma unroll
        for (int e = 0; e < kMaxPosReg; ++e) {
          const int64_t l = (int64_t)pos[t][e] - l0;
          if (pos[t][e] >= 0 && l >= 0 && l < CH) ym |= 1u << l;
        }
        for (int e = kMaxPosReg; e < npos[t]; ++e) {  // rows with many positives
          const int64_t l = (int64_t)a.pos_ids[pbeg[t] + e] - l0;
          if (l >= 0 && l < CH) ym |= 1u << l;
        }
#pragma unroll
        for (int c = 0; c < CH; c += 16) {
          const float* z = &zall[t][c];
          // y = 0 everywhere first (positives are rare), then the few positive
          // columns are corrected: dY -= scale, loss -= z.
          float dyv[16], relu = 0.f, prod = 1.f;
#pragma unroll
          for (int e = 0; e < NC; ++e) {
            const float th = tanh_approx(0.5f * z[e]);   // sigma(z) = (1 + th) / 2
            dyv[e] = fmaf(hs, th, hs);                   // scale * sigma(z)
            relu += fmaxf(z[e], 0.f);
            prod *= fmaf(0.5f, fabsf(th), 0.5f);         // sigma(|z|)
          }
          float zy = 0.f;
          const uint32_t yc = (ym >> c) & ((1u << NC) - 1u);
          if (yc) {
#pragma unroll
            for (int e = 0; e < NC; ++e)
              if ((yc >> e) & 1u) {
                dyv[e] -= sl;
                zy += z[e];
              }
          }
          // softplus(z) - z y = max(z, 0) - log sigma(|z|) - z y
          if (live) loss_acc += relu - zy - __logf(prod);
#pragma unroll
          for (int hq = 0; hq < NC / 8; ++hq) {
            const uint4 v = make_uint4(pack_bf16x2(dyv[8 * hq], dyv[8 * hq + 1]),
                                       pack_bf16x2(dyv[8 * hq + 2], dyv[8 * hq + 3]),
                                       pack_bf16x2(dyv[8 * hq + 4], dyv[8 * hq + 5]),
                                       pack_bf16x2(dyv[8 * hq + 6], dyv[8 * hq + 7]));
            const int col = hh * CH + c + 8 * hq;
            *reinterpret_cast<uint4*>(dyrow + swz_rows((uint32_t)(b * RB + col * 2), RB)) = v;  // rows past B: zeros
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dy_full[s]);
      return true;
    };
    auto readout = [&](int i) -> bool {
      const int64_t g = gb + i;
      const int s = i & 1;
      // the update's first W and momentum values do not depend on dW: their loads
      // are in flight while the dW product finishes
      constexpr int NC0 = CH < 16 ? CH : 16;
      float wv0[NC0], mv0[NC0];
      if constexpr (kUpd > 0) {
        if (r < kK) {
          const int64_t o = (g * kG + hh * CH) * kK + r;
#pragma unroll
          for (int e = 0; e < NC0; ++e) {
            wv0[e] = __bfloat162float(W[o + (int64_t)e * kK]);
            mv0[e] = kUpd == 2 ? __bfloat162float(a.M[o + (int64_t)e * kK]) : 0.f;
          }
        }
      }
      if (!wait_or_abort(&dw_full[s], (i >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      // dW readout: row = slot r, columns = this warp's labels (all requested before the wait)
      constexpr int NCR = CH < 16 ? CH : 16;
      float vall[CH];
#pragma unroll
      for (int c = 0; c < CH; c += 16) {
        if constexpr (NCR == 8) tmem_ld8(D(s) + lane_off + (uint32_t)(hh * CH + c), &vall[c]);
        else tmem_ld16(D(s) + lane_off + (uint32_t)(hh * CH + c), *reinterpret_cast<float(*)[16]>(&vall[c]));
      }
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < CH; c += 16) {
        constexpr int NC = NCR;
        const float* v = &vall[c];
        if (r < kK) {
          const int64_t off0 = (g * kG + hh * CH + c) * kK + r;  // (label, slot r); lanes: consecutive slots
          if constexpr (kUpd == 0) {
#pragma unroll
            for (int e = 0; e < NC; ++e) a.dW[off0 + (int64_t)e * kK] = __float2bfloat16_rn(v[e]);
          } else {
            float wv[16], mv[16];
#pragma unroll
            for (int e = 0; e < NC; ++e) {
              if (c == 0) {
                wv[e] = wv0[e];
                mv[e] = mv0[e];
              } else {
                wv[e] = __bfloat162float(W[off0 + (int64_t)e * kK]);
                mv[e] = kUpd == 2 ? __bfloat162float(a.M[off0 + (int64_t)e * kK]) : 0.f;
              }
            }
#pragma unroll
            for (int e = 0; e < NC; ++e) {
              const float m = kUpd == 2 ? fmaf(a.momentum, mv[e], v[e]) : v[e];
              if constexpr (kUpd == 2) a.M[off0 + (int64_t)e * kK] = __float2bfloat16_rn(m);
              a.W_out[off0 + (int64_t)e * kK] = __float2bfloat16_rn(fmaf(-a.lr, m, wv[e]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[s]);
      return true;
    };
    bool ok = n_items > 0 ? bce(0) : true;
    for (int i = 0; ok && i < n_items; ++i) {
      if (i + 1 < n_items && !bce(i + 1)) break;
      if (!readout(i)) break;
    }
    // deterministic loss reduction over the epilogue warps (named barrier 1)
    float v = loss_acc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[ew] = v;
    named_bar(1, 32 * kStepEpi);
    if (ew == 0 && lane == 0) {
      float t = 0.f;
      for (int j = 0; j < kStepEpi; ++j) t += red[j];
      a.loss_part[blockIdx.x] = t;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == kStepMma) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace v2

// ------------------------------------------------------------- host side
namespace tail2 {

bool supported(int G, int k, int Bp) {
  return (G == 16 || G == 32 || G == 64) && (k == 64 || k == 128) && Bp <= 256;
}

size_t step_smem(int Bp, int k, int G) { return v2::step_layout(Bp, k, G).total; }
cudaError_t tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer);
template <int kG, int kK, int kUpd>
cudaError_t launch_step_t(const v2::StepArgs& a, int grid, const void* Xt, const void* W, cudaStream_t st) {
  const size_t smem = step_smem(a.sh.Bp, kK, kG);
  auto kern = v2::k_step2<kG, kK, kUpd>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // the gradient buffer [n_items * Bp][64] as the stores' tensor: group g's box
  // (G labels x Bp rows) at columns (g % NG) * G of item g / NG's rows, NG = 64 / G
  CUtensorMap tm_dy;
  const uint64_t n_items = (uint64_t)(a.sh.n_groups + 64 / kG - 1) / (64 / kG);
  e = tmap_2d(&tm_dy, a.dY_out, 64, n_items * a.sh.Bp, 128, kG, (uint32_t)a.sh.Bp);
  if (e != cudaSuccess) return e;
  kern<<<grid, v2::kStepThreads, smem, st>>>(a, static_cast<const __nv_bfloat16*>(Xt),
                                             static_cast<const __nv_bfloat16*>(W), tm_dy);
  return cudaGetLastError();
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D bf16 tensor map: `inner` contiguous elements per row, `outer` rows of
// `row_bytes` bytes; box of box_inner x box_outer elements, read past the edges as
// zeros.  The swizzle follows the box row width (32, 64 or 128 bytes).
cudaError_t tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return cudaErrorNotSupported;
  const uint32_t rb = box_inner * 2;
  const CUtensorMapSwizzle sw = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                           : CU_TENSOR_MAP_SWIZZLE_32B;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

#define HASTE_V2_DISPATCH(FN, ...)                                     \
  switch (G * 1000 + k) {                                              \
    case 16064: return FN<16, 64>(__VA_ARGS__);                        \
    case 16128: return FN<16, 128>(__VA_ARGS__);                       \
    case 32064: return FN<32, 64>(__VA_ARGS__);                        \
    case 32128: return FN<32, 128>(__VA_ARGS__);                       \
    case 64064: return FN<64, 64>(__VA_ARGS__);                        \
    case 64128: return FN<64, 128>(__VA_ARGS__);                       \
    default: return cudaErrorInvalidValue;                             \
  }

template <int kG, int kK>
cudaError_t launch_step_dw(const v2::StepArgs& a, int grid, const void* Xt, const void* W, cudaStream_t st) {
  return launch_step_t<kG, kK, 0>(a, grid, Xt, W, st);
}
template <int kG, int kK>
cudaError_t launch_step_sgd(const v2::StepArgs& a, int grid, const void* Xt, const void* W, cudaStream_t st) {
  return launch_step_t<kG, kK, 1>(a, grid, Xt, W, st);
}
template <int kG, int kK>
cudaError_t launch_step_sgdm(const v2::StepArgs& a, int grid, const void* Xt, const void* W, cudaStream_t st) {
  return launch_step_t<kG, kK, 2>(a, grid, Xt, W, st);
}

// upd: 0 writes dW; 1 applies SGD (W' = W - lr dW); 2 SGD with momentum.
cudaError_t launch_step(int G, int k, int upd, const v2::StepArgs& a, int grid, const void* Xt, const void* W,
                        cudaStream_t st) {
  if (upd == 1) {
    HASTE_V2_DISPATCH(launch_step_sgd, a, grid, Xt, W, st)
  } else if (upd == 2) {
    HASTE_V2_DISPATCH(launch_step_sgdm, a, grid, Xt, W, st)
  }
  HASTE_V2_DISPATCH(launch_step_dw, a, grid, Xt, W, st)
}

}  // namespace tail2
}  // namespace haste
