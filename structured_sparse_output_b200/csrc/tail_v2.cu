// tail_v2.cu -- warp-specialised, pipelined bf16 kernels of the group-shared sparse
// tail (HASTE, "Hardware-Aware Dynamic Sparse Training for Large Output Spaces",
// Methodology 1: labels in groups of G share one fan-in set I_g of k features).
//
// k_step2 -- fused forward + BCE gradient + dW, one group per iteration, with the
// group's labels as the small M of weight-stationary MMAs (MW = 32 rows for G <= 32,
// 64 for G = 64), so that one instruction covers the whole batch (forward: N = Bp)
// or every slot (dW: N = k):
//   forward  logits_g^T [MW, Bp] = W_g [MW, k] . Xg^T     (K = k)
//   dW       dW_g^T     [MW, k]  = dY_g^T [MW, Bp] . Xg   (K = Bp)
//   warps 0, 12  MMA issuers (one thread each): warp 0 issues each group's
//              forward, warp 12 its dW product, each as soon as its inputs are
//              ready (in the narrow block of the G = 64 update kernels warp 0
//              issues both);
//   producers  six warps (three in the narrow block): the gather-once tile Xg = X[:, I_g]
//              (k rows of X^T) and the G x k weight block, staged with cp.async
//              into a 2-stage ring (all of them fill the stage of each group);
//   epilogue   eight warps: each thread owns one label and a run of batch rows of the
//              logits; they leave TMEM only as the BCE gradient dY^T (bf16, into
//              shared memory: the dW operand, and the tile that epilogue thread 0
//              writes to the gradient buffer of the dX pass with TMA stores).  The
//              positives of the group come from a per-row cursor over the sorted
//              CSR targets, turned into label x row bit masks in shared memory.
//              The BCE of group i+1 comes before the dW readout of group i, so the
//              dW product runs behind it.  The readout writes dW as 32-byte
//              (or 16-byte) vectors of one label row, or (kUpd > 0) applies an
//              SGD update to the group's weights while dW is on chip:
//              M' = momentum * M + dW (kUpd = 2) or M' = dW (kUpd = 1),
//              W' = W - lr * M', with W' written to a separate buffer (the dX pass
//              still reads W) and M' over M.
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
  __nv_bfloat16* dY_out;  // gradient buffer of the dX pass: [n_items * 64][Bp], label rows
  float* loss_part;
  const int32_t* pos_ptr;
  const int32_t* pos_ids;
  float grad_scale;
  int out_v8;  // the readout's outputs (dW, or W_out and M) are 32-byte aligned: 32-byte stores
};

// Rows of the weight-stationary MMAs for groups of G labels.
__host__ __device__ constexpr int step_mw(int G) { return G <= 32 ? 32 : 64; }

// ------------------------------------------------------------ smem layouts
// Per stage: Xg [Bp/64][k][64] (slot rows, 64 batch columns per 128-byte row),
// W_g [k/64][MW][64] (label rows, 64 slots per row) and dY^T [Bp/64][MW][64]
// (label rows, 64 batch columns per row), all 128B-swizzled, and the group's
// positive-label bit masks [Bp/32][MW]: their own space for MW = 32, for MW = 64
// (no room left) the W_g space once the forward has read it.
struct StepLayout {
  uint32_t xg[2], wg[2], dy[2], mk[2], bars, total;
};
__host__ __device__ inline StepLayout step_layout(int Bp, int k, int G) {
  StepLayout L;
  const int MW = step_mw(G);
  const uint32_t xg = (uint32_t)((Bp / 64) * k * 128);
  const uint32_t wg = (uint32_t)((k / 64) * MW * 128);
  const uint32_t dy = (uint32_t)((Bp / 64) * MW * 128);
  uint32_t off = 0;
  for (int s = 0; s < 2; ++s) { L.xg[s] = off; off += xg; }
  for (int s = 0; s < 2; ++s) { L.wg[s] = off; off += wg; }
  for (int s = 0; s < 2; ++s) { L.dy[s] = off; off += dy; }
  for (int s = 0; s < 2; ++s) {
    if (MW == 32) {
      L.mk[s] = off;
      off += (uint32_t)((Bp / 32) * MW * 4);
    } else {
      L.mk[s] = L.wg[s];
    }
  }
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

// 32 lanes x 32 consecutive 32-bit TMEM columns (two x16 loads; one wait after).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(v));
  tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(v + 16));
}

// ============================================================ k_step2
// Warp roles (warp w runs on scheduler w % 4, which also fixes the TMEM lane
// quarter an epilogue warp can read).  The MMA issuers (warps 0 and 12) share
// their scheduler with no producer: the producers' stream of cp.async fills the
// memory-instruction queue of theirs, and each barrier test of an issuer would
// wait behind it.
//   wide block (512 threads): warp 0 issues the forwards, warp 12 the dW
//            products; six producer warps (1-3, 5-7, two on each of schedulers
//            1-3) keep more gathered rows in flight; epilogue warps 4 and 8
//            (quarter 0), 9 and 13 (1), 10 and 14 (2), 11 and 15 (3).
//   narrow block (384 threads, G = 64 with the SGD update, whose epilogue needs
//            the registers): warp 0 issues both kinds, three producer warps
//            (1-3), epilogue warps 4-11.
constexpr int kStepMma = 0;        // warp id of the forward issuer
constexpr int kStepMmaW = 12;      // warp id of the dW issuer
constexpr int kStepEpi = 8;        // epilogue warps: 4 lane quarters x 2 column halves
constexpr int kStepEpiThreads = 32 * kStepEpi;
// The wide block (16 warps) for every kernel but the G = 64 update kernels, whose
// 64-label epilogue with the SGD update needs the registers of a 12-warp block.
__host__ __device__ constexpr bool step_wide(int G, int upd) { return !(G == 64 && upd > 0); }
__host__ __device__ constexpr int step_prod_warps(bool wide) { return wide ? 6 : 3; }
__host__ __device__ constexpr int step_threads(bool wide) { return wide ? 32 * 16 : 32 * 12; }
// producer index of warp w (-1: not a producer)
template <bool kWide>
__device__ __forceinline__ int step_prod_part(int w) {
  if constexpr (kWide) return w >= 1 && w <= 3 ? w - 1 : w >= 5 && w <= 7 ? w - 2 : -1;
  else return w >= 1 && w <= 3 ? w - 1 : -1;
}
// epilogue index ew = quarter + 4 * half of warp w (-1: not an epilogue warp)
template <bool kWide>
__device__ __forceinline__ int step_epi_index(int w) {
  if constexpr (kWide) return w == 4 ? 0 : w == 8 ? 4 : w >= 9 && w != 12 ? w - 8 : -1;
  else return w >= 4 && w <= 11 ? w - 4 : -1;
}

template <int kG, int kK, int kUpd>
__global__ void __launch_bounds__(step_threads(step_wide(kG, kUpd)), 1)
    k_step2(StepArgs a, const __nv_bfloat16* __restrict__ Xt, const __nv_bfloat16* __restrict__ W,
            const __grid_constant__ CUtensorMap tm_dy) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int MW = step_mw(kG);     // rows of the weight-stationary MMAs
  constexpr bool kWide = step_wide(kG, kUpd);
  constexpr int NGI = 64 / kG;        // groups per 64-label item of the gradient buffer
  const TailShape sh = a.sh;
  const int Bp = sh.Bp;
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
      mbar_init(&full[s], 32 * step_prod_warps(kWide));
      mbar_init(&empty[s], 1);
      mbar_init(&fwd_full[s], 1);
      mbar_init(&dy_full[s], kStepEpi);
      mbar_init(&dw_full[s], 1);
      mbar_init(&tmem_empty[s], kStepEpi);
    }
    mbar_init(done, kWide ? 2 : 1);
    // A limit below one sleep, set only to exercise the abort paths, makes the
    // first wait of every warp run out at once (the waits themselves read the
    // limit only after their first, blocking test: a short limit would not make a
    // wait whose phase completes within that test run out).
    if (g_wait_limit_ns < kWaitSuspendNs) {
      *abort_flag = 1;
      record_error(kErrTimeout);
    } else {
      *abort_flag = 0;
    }
    fence_mbar_init();
  }
  // TMEM: logits^T accumulators F[2] (Bp columns over the lane quarters: Bp/4 for
  // MW = 32, Bp/2 for MW = 64), dW^T accumulators D[2] (k/4 or k/2 columns)
  const uint32_t f_cols = (uint32_t)(MW == 32 ? Bp / 4 : Bp / 2);
  constexpr uint32_t d_cols = MW == 32 ? kK / 4 : kK / 2;
  const uint32_t ncols = tmem_cols_for(2 * f_cols + 2 * d_cols);
  if (w == kStepMma) {
    tmem_alloc(tslot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  auto F = [&](int s) -> uint32_t { return tmem + (s ? f_cols : 0u); };
  auto D = [&](int s) -> uint32_t { return tmem + 2 * f_cols + (s ? d_cols : 0u); };
  auto XG = [&](int s) -> uint32_t { return base + (s ? Lo.xg[1] : Lo.xg[0]); };
  auto WG = [&](int s) -> uint32_t { return base + (s ? Lo.wg[1] : Lo.wg[0]); };
  auto DY = [&](int s) -> uint32_t { return s ? Lo.dy[1] : Lo.dy[0]; };

  // contiguous chunk of groups per CTA
  const int64_t gb = (int64_t)blockIdx.x * sh.n_groups / gridDim.x;
  const int64_t ge = (int64_t)(blockIdx.x + 1) * sh.n_groups / gridDim.x;
  const int n_items = (int)(ge - gb);

  if (step_prod_part<kWide>(w) >= 0) {
    // ------------------------------------------------- cp.async producers
    // the producer warps fill the stage of every item i (stage i & 1); warp part
    // copies the groups of four rows part, part + P, ...  Lane (rg, sub) copies
    // the 16-byte chunk sub of every 128-byte segment of its rows, so that 8
    // consecutive lanes read one segment; the feature indices of its rows sit in
    // registers.
    constexpr int P = step_prod_warps(kWide);
    constexpr int kQuads = kK / 4;                 // groups of four rows
    constexpr int kRows = (kQuads + P - 1) / P;    // per warp (the last may be short)
    const int part = step_prod_part<kWide>(w), ht = lane;
    const int sub = ht & 7, rg = ht >> 3;
    for (int i = 0; i < n_items; ++i) {
      const int64_t g = gb + i;
      const int half = i & 1;
      const uint32_t xg = XG(half), wg = WG(half);
      // the group after next: weight block and indices into L2 (from HBM they
      // would stretch the gather of that group)
      if (part == 0 && lane == 0 && i + 2 < n_items) {
        prefetch_l2(W + (g + 2) * kG * kK, (uint32_t)(kG * kK * 2));
        prefetch_l2(a.idx + (g + 2) * kK, (uint32_t)(kK * 4));
        if constexpr (kUpd == 2) prefetch_l2(a.M + (g + 2) * kG * kK, (uint32_t)(kG * kK * 2));  // read by the update
      }
      // the index loads are in flight while this half waits for its stage
      int idx_cur[kRows];
#pragma unroll
      for (int m = 0; m < kRows; ++m)
        idx_cur[m] = m * P + part < kQuads ? a.idx[g * kK + rg + 4 * (m * P + part)] : 0;
      if (!wait_or_abort(&empty[half], ((i >> 1) & 1) ^ 1, abort_flag)) break;
      const int nbb = Bp / 64;
#pragma unroll
      for (int m = 0; m < kRows; ++m) {
        if (m * P + part >= kQuads) break;
        const int sl = rg + 4 * (m * P + part);
        const __nv_bfloat16* src = Xt + (int64_t)idx_cur[m] * Bp + sub * 8;
        const uint32_t dst = xg + sw128((uint32_t)(sl * 128 + sub * 16));  // swizzle is the same in every block
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
          if (bb < nbb) cp_async16(dst + (uint32_t)(bb * kK * 128), src + bb * 64, 16);
      }
      // weight block of the group (contiguous G x k) into label rows of MW-row
      // blocks of 64 slots; chunks split between the warps
      const __nv_bfloat16* wsrc = W + g * (int64_t)kG * kK;
      constexpr int cpr = kK / 8;
#pragma unroll 4
      for (int c0 = 32 * part; c0 < kG * cpr; c0 += 32 * P) {
        const int c = c0 + ht;
        const int j = c / cpr, cc = c % cpr;
        cp_async16(wg + sw128((uint32_t)((cc >> 3) * MW * 128 + j * 128 + (cc & 7) * 16)),
                   wsrc + (int64_t)j * kK + cc * 8, 16);
      }
      cp_async_commit();
      publish_all(&full[half]);
    }
    cp_async_wait_all();
  } else if (w == kStepMma || (kWide && w == kStepMmaW)) {
    // ------------------------------------------------------------ MMA issuers
    // Wide block: two warps, each sleeping in the barrier it waits for (no polling
    // loop over both kinds, so each wakes as soon as its operands are ready; on the
    // step of 670K labels this is 6% faster), one thread of each issuing:
    //   warp kStepMma:  forward of group i once its stage is loaded (full) and
    //                   F(i&1) is free (the BCE of group i - 2 has read it:
    //                   dy_full).  A = W_g (K-major, label rows), B = Xg
    //                   (MN-major: batch contiguous, 64-column blocks kK*128
    //                   bytes apart), K = 16 slots;
    //   warp kStepMmaW: dW of group i once its BCE is done (dy_full) and D(i&1)
    //                   has been read out for group i - 2 (tmem_empty).
    //                   A = dY^T (K-major, label rows), B = Xg (K-major: slot
    //                   rows), K = 16 batch rows; its commits free the readout
    //                   (dw_full) and the stage (empty).
    // A wait that runs out raises the abort flag; the other waits then fail fast.
    // Descriptors advance by constant start-address offsets (16-byte units).
    if constexpr (kWide) {
      if (w == kStepMma) {
        const uint32_t idesc_f = make_idesc(1, 0, 1, MW, (uint32_t)Bp);
        for (int i = 0; i < n_items; ++i) {
          const int s = i & 1;
          if (!__all_sync(0xffffffffu, wait_or_abort(&full[s], (i >> 1) & 1, abort_flag))) break;
          if (i >= 2 && !__all_sync(0xffffffffu, wait_or_abort(&dy_full[s], ((i - 2) >> 1) & 1, abort_flag))) break;
          if (lane == 0) {
            tc_fence_after();
            const uint64_t ad0 = make_sdesc(WG(s), 16, 1024, kLayoutSw128);
            const uint64_t bd0 = make_sdesc(XG(s), (uint32_t)kK * 128, 1024, kLayoutSw128);
            const uint32_t f = F(s);
#pragma unroll
            for (int kk = 0; kk < kK / 16; ++kk)
              mma_ws(f, ad0 + (uint64_t)(((kk / 4) * MW * 128 + (kk % 4) * 32) >> 4), bd0 + (uint64_t)(kk * 128),
                     idesc_f, kk > 0 ? 1u : 0u);
            mma_commit(&fwd_full[s]);
          }
          __syncwarp();
        }
      } else {
        const uint32_t idesc_w = make_idesc(1, 0, 0, MW, kK);
        for (int i = 0; i < n_items; ++i) {
          const int s = i & 1;
          if (!__all_sync(0xffffffffu, wait_or_abort(&dy_full[s], (i >> 1) & 1, abort_flag))) break;
          if (!__all_sync(0xffffffffu, wait_or_abort(&tmem_empty[s], ((i >> 1) & 1) ^ 1, abort_flag))) break;
          if (lane == 0) {
            tc_fence_after();
            const uint64_t ad0 = make_sdesc(base + DY(s), 16, 1024, kLayoutSw128);
            const uint64_t bd0 = make_sdesc(XG(s), 16, 1024, kLayoutSw128);
            const uint32_t d = D(s);
            auto dw_mma = [&](int kk) {
              mma_ws(d, ad0 + (uint64_t)(((kk / 4) * MW * 128 + (kk % 4) * 32) >> 4),
                     bd0 + (uint64_t)(((kk / 4) * kK * 128 + (kk % 4) * 32) >> 4), idesc_w, kk > 0 ? 1u : 0u);
            };
            if (Bp == 256) {
#pragma unroll
              for (int kk = 0; kk < 16; ++kk) dw_mma(kk);
            } else {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) dw_mma(kk);
            }
            mma_commit(&dw_full[s]);
            mma_commit(&empty[s]);
          }
          __syncwarp();
        }
      }
    } else {
      // Narrow block: warp 0 issues both kinds.
      // Forwards and dW products are issued as their inputs become ready, not in a
      // fixed interleave: fwd(j) needs its gathered stage (full) and F(j&1) free,
      // which holds once dW(j-2) was issued (its BCE had finished reading F);
      // dW(j) needs the BCE of j (dy_full) and D(j&1) read out for j-2
      // (tmem_empty).  Lane 0 polls; the decisions are broadcast so the warp stays
      // converged.  No progress for the wait limit raises the abort flag.
      //   forward: A = W_g (K-major, label rows), B = Xg (MN-major: batch
      //            contiguous, 64-column blocks kK*128 bytes apart), K = 16 slots;
      //   dW:      A = dY^T (K-major, label rows), B = Xg (K-major: slot rows),
      //            K = 16 batch rows.
      const uint32_t idesc_f = make_idesc(1, 0, 1, MW, (uint32_t)Bp);
      const uint32_t idesc_w = make_idesc(1, 0, 0, MW, kK);
      int nf = 0, nd = 0;
      // the timer is read only while nothing is ready, and then once every 64 polls
      // (a read costs hundreds of cycles, which would delay the next issue): t_idle
      // is when the current idle stretch began, 0 after progress
      uint64_t t_idle = 0;
      uint32_t idle_polls = 0;
      const uint64_t limit = g_wait_limit_ns;
      while (nd < n_items) {
        bool did = false;
        if (nf < n_items && nf <= nd + 1) {
          const int s = nf & 1;
          const bool rdy = __shfl_sync(0xffffffffu, lane == 0 ? mbar_test_wait(&full[s], (nf >> 1) & 1) : false, 0);
          if (rdy) {
            if (lane == 0) {
              tc_fence_after();
              // descriptors advance by constant start-address offsets (16-byte units):
              // the issuing warp shares its scheduler with busy warps, so each MMA
              // costs only a few instructions
              const uint64_t ad0 = make_sdesc(WG(s), 16, 1024, kLayoutSw128);
              const uint64_t bd0 = make_sdesc(XG(s), (uint32_t)kK * 128, 1024, kLayoutSw128);
              const uint32_t f = F(s);
#pragma unroll
              for (int kk = 0; kk < kK / 16; ++kk)
                mma_ws(f, ad0 + (uint64_t)(((kk / 4) * MW * 128 + (kk % 4) * 32) >> 4), bd0 + (uint64_t)(kk * 128), idesc_f,
                       kk > 0 ? 1u : 0u);
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
                                       lane == 0 ? (mbar_test_wait(&dy_full[s], (nd >> 1) & 1) &&
                                                    mbar_test_wait(&tmem_empty[s], ((nd >> 1) & 1) ^ 1))
                                                 : false,
                                       0);
          if (rdy) {
            if (lane == 0) {
              tc_fence_after();
              const uint64_t ad0 = make_sdesc(base + DY(s), 16, 1024, kLayoutSw128);
              const uint64_t bd0 = make_sdesc(XG(s), 16, 1024, kLayoutSw128);
              const uint32_t d = D(s);
              auto dw_mma = [&](int kk) {
                mma_ws(d, ad0 + (uint64_t)(((kk / 4) * MW * 128 + (kk % 4) * 32) >> 4),
                       bd0 + (uint64_t)(((kk / 4) * kK * 128 + (kk % 4) * 32) >> 4), idesc_w, kk > 0 ? 1u : 0u);
              };
              if (Bp == 256) {
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) dw_mma(kk);
              } else {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) dw_mma(kk);
              }
              mma_commit(&dw_full[s]);
              mma_commit(&empty[s]);
            }
            __syncwarp();
            ++nd;
            did = true;
          }
        }
        if (did) {
          t_idle = 0;
          idle_polls = 0;
        } else {
          if (*abort_flag) break;
          if ((idle_polls++ & 63u) == 0) {
            const uint64_t now = globaltimer_ns();
            if (t_idle == 0) t_idle = now;
            if (now - t_idle > limit) {
              if (lane == 0) {
                *abort_flag = 1;
                record_error(kErrTimeout);
              }
              __syncwarp();
              break;
            }
          }
          // no sleep here: a suspended issuer wakes far later than the barriers
          // complete, and the tensor core would wait for it
        }
      }
    }
    // Also after an abort: the CTA frees TMEM and exits only once every MMA its
    // issuers issued has finished writing TMEM and reading shared memory.
    if (lane == 0) mma_commit(done);
    __syncwarp();
    (void)__all_sync(0xffffffffu, mbar_wait(done, 0));
  } else if (step_epi_index<kWide>(w) >= 0) {
    // ------------------------------------------------------------- epilogue
    // warp (q, hh): TMEM lane quarter q, half hh of the quarter's columns
    const int ew = step_epi_index<kWide>(w), q = w & 3, hh = ew >> 2;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    // this thread's label m (a row of the MW-row products), its run of nct batch
    // rows from b0 (logits) and of NSL slots from s0 (dW)
    const int m = MW == 32 ? lane : (q & 1) * 32 + lane;
    const bool mvalid = m < kG;
    const int nct = (int)f_cols / 2;
    const int b0 = (MW == 32 ? q * (Bp / 4) : (q >> 1) * (Bp / 2)) + hh * nct;
    constexpr int NSL = (int)d_cols / 2;
    constexpr int NCT_MAX = MW == 32 ? 32 : 64;
    const int s0 = (MW == 32 ? q * (kK / 4) : (q >> 1) * (kK / 2)) + hh * NSL;
    const float scale = a.grad_scale, hs = 0.5f * scale;
    const int live = min(nct, sh.B - b0);  // rows of the run below B (may be <= 0)
    float loss_acc = 0.f;
    // cursor of batch row rb over its positives (ids ascending): the first one at or
    // after the current group's first label
    const int rb = ew * 32 + lane;
    int cur = 0, cend = 0, nid = INT_MAX;
    if (rb < sh.B) {
      cur = a.pos_ptr[rb];
      cend = a.pos_ptr[rb + 1];
      const int first = (int)(gb * kG);
      int lo = cur, hi = cend;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a.pos_ids[mid] < first) lo = mid + 1;
        else hi = mid;
      }
      cur = lo;
      nid = cur < cend ? a.pos_ids[cur] : INT_MAX;
    }
    // Bit masks of group i's positives into the W_g space of its stage (free once
    // the forward has read it): word [warp w'][label j] holds bit l for batch row
    // 32 w' + l.  Each warp writes only its own words, whole.
    auto build = [&](int i) {
      const int lo = (int)((gb + i) * kG), hi = lo + kG;
      uint64_t lm = 0;  // labels of the group that are positive in row rb
      while (nid < hi) {
        if (nid >= lo) lm |= 1ull << (nid - lo);
        ++cur;
        nid = cur < cend ? a.pos_ids[cur] : INT_MAX;
      }
      const uint32_t any_lo = __reduce_or_sync(0xffffffffu, (uint32_t)lm);
      const uint32_t any_hi = MW == 64 ? __reduce_or_sync(0xffffffffu, (uint32_t)(lm >> 32)) : 0u;
      uint32_t w0 = 0, w1 = 0;
      for (uint32_t r = any_lo; r; r &= r - 1) {
        const int j = __ffs(r) - 1;
        const uint32_t bj = __ballot_sync(0xffffffffu, (uint32_t)(lm >> j) & 1u);
        if (j == lane) w0 = bj;
      }
      for (uint32_t r = any_hi; r; r &= r - 1) {
        const int j = __ffs(r) - 1;
        const uint32_t bj = __ballot_sync(0xffffffffu, (uint32_t)(lm >> (32 + j)) & 1u);
        if (j == lane) w1 = bj;
      }
      if (ew * 32 < Bp) {
        uint32_t* mk = reinterpret_cast<uint32_t*>(gbase + Lo.mk[i & 1]) + ew * MW;
        mk[lane] = w0;
        if constexpr (MW == 64) mk[32 + lane] = w1;
      }
    };
    // group i's dY^T tile to the dX pass's buffer (epilogue thread 0, once every
    // epilogue warp has written it): the G label rows of its item (64 / G
    // consecutive groups, 64 labels), one box per 64 batch columns
    const bool storer = ew == 0 && lane == 0;
    auto store_dy = [&](int i) {
      const int64_t g = gb + i;
      const int row0 = (int)((g / NGI) * 64 + (g % NGI) * kG);
      for (int blk = 0; blk < Bp / 64; ++blk)
        tma_store_2d(&tm_dy, base + DY(i & 1) + (uint32_t)(blk * MW * 128), 64 * blk, row0);
      bulk_commit();
    };
    // BCE of group i: false (the same in every epilogue thread) when the epilogue
    // stops, after a wait ran out earlier.  Its barrier also orders the stores: the
    // tile of group i - 2 (this stage) has been read before anyone writes the stage
    // again, and group i - 1's tile is complete when it is stored.
    auto bce = [&](int i, bool& failed) -> bool {
      const int s = i & 1;
      // With their own mask space (MW = 32), the masks, the barrier and the
      // previous group's stores do not depend on the forward and run while it does;
      // for MW = 64 the masks take the W_g space after the forward.  A wait that runs
      // out stops the loop at the next barrier (every warp passes the same barriers).
      if constexpr (MW == 64) {
        if (!failed && !__all_sync(0xffffffffu, wait_or_abort(&fwd_full[s], (i >> 1) & 1, abort_flag))) failed = true;
      }
      if (!failed) build(i);
      if (storer) bulk_wait_read<0>();
      if (named_bar_or(1, kStepEpiThreads, failed || *abort_flag)) return false;
      if (storer && i >= 1) store_dy(i - 1);
      if constexpr (MW == 32) {
        if (!__all_sync(0xffffffffu, wait_or_abort(&fwd_full[s], (i >> 1) & 1, abort_flag))) {
          failed = true;
          return true;
        }
      }
      tc_fence_after();
      float z[NCT_MAX];
#pragma unroll
      for (int c = 0; c < NCT_MAX; c += 16)
        if (c < nct) tmem_ld16(F(s) + lane_off + (uint32_t)(hh * nct + c), *reinterpret_cast<float(*)[16]>(&z[c]));
      tmem_wait_ld();
      const uint32_t* mk = reinterpret_cast<const uint32_t*>(gbase + Lo.mk[s]);
      uint64_t ym = mk[(b0 >> 5) * MW + m];
      if (nct > 32) ym |= (uint64_t)mk[((b0 >> 5) + 1) * MW + m] << 32;
      ym >>= (b0 & 31);
      uint8_t* dyt = gbase + DY(s);
#pragma unroll
      for (int c = 0; c < NCT_MAX; c += 16) {
        if (c >= nct) break;
        // y = 0 everywhere first (positives are rare), then the few positive
        // rows are corrected: dY -= scale, loss -= z
        float dyv[16], relu = 0.f, prod = 1.f, zy = 0.f;
        if (c + 16 <= live) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float th = tanh_approx(0.5f * z[c + e]);  // sigma(z) = (1 + th) / 2
            dyv[e] = fmaf(hs, th, hs);                      // scale * sigma(z)
            relu += fmaxf(z[c + e], 0.f);
            prod *= fmaf(0.5f, fabsf(th), 0.5f);            // sigma(|z|)
          }
        } else {  // the run reaches past B: those rows get dY = 0 and no loss
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const bool lv = c + e < live;
            const float th = tanh_approx(0.5f * z[c + e]);
            dyv[e] = lv ? fmaf(hs, th, hs) : 0.f;
            relu += lv ? fmaxf(z[c + e], 0.f) : 0.f;
            prod *= lv ? fmaf(0.5f, fabsf(th), 0.5f) : 1.f;
          }
        }
        const uint32_t yc = (uint32_t)(ym >> c) & 0xFFFFu;
        if (yc) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if ((yc >> e) & 1u) {
              dyv[e] -= scale;
              zy += z[c + e];
            }
        }
        // softplus(z) - z y = max(z, 0) - log sigma(|z|) - z y
        if (mvalid) loss_acc += relu - zy - __logf(prod);
        const int b = b0 + c;
        const uint32_t row = (uint32_t)((b >> 6) * MW * 128 + m * 128);
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const uint4 v = make_uint4(pack_bf16x2(dyv[8 * hq], dyv[8 * hq + 1]), pack_bf16x2(dyv[8 * hq + 2], dyv[8 * hq + 3]),
                                     pack_bf16x2(dyv[8 * hq + 4], dyv[8 * hq + 5]),
                                     pack_bf16x2(dyv[8 * hq + 6], dyv[8 * hq + 7]));
          *reinterpret_cast<uint4*>(dyt + sw128(row + (uint32_t)((((b & 63) >> 3) + hq) * 16))) = v;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dy_full[s]);
      return true;
    };
    // dW readout of group i: this thread's label row, NSL consecutive slots, as
    // 16-byte vectors.  False (the same in the whole warp) when a wait ran out.
    auto readout = [&](int i) -> bool {
      const int s = i & 1;
      const int64_t o = ((gb + i) * kG + m) * kK + s0;  // dW[label][slot s0]
      // the update's W and momentum values do not depend on dW: their loads are in
      // flight while the dW product finishes
      uint4 wv[NSL / 8], mv[NSL / 8];
      if constexpr (kUpd > 0) {
        if (mvalid) {
#pragma unroll
          for (int c = 0; c < NSL / 8; ++c) {
            wv[c] = *reinterpret_cast<const uint4*>(W + o + 8 * c);
            mv[c] = kUpd == 2 ? *reinterpret_cast<const uint4*>(a.M + o + 8 * c) : make_uint4(0, 0, 0, 0);
          }
        }
      }
      if (!__all_sync(0xffffffffu, wait_or_abort(&dw_full[s], (i >> 1) & 1, abort_flag))) return false;
      tc_fence_after();
      float v[NSL];
#pragma unroll
      for (int c = 0; c < NSL; c += 16) {
        if constexpr (NSL == 8) tmem_ld8(D(s) + lane_off + (uint32_t)(hh * NSL), v);
        else tmem_ld16(D(s) + lane_off + (uint32_t)(hh * NSL + c), *reinterpret_cast<float(*)[16]>(&v[c]));
      }
      tmem_wait_ld();
      bool stored = false;
      if constexpr (NSL % 16 == 0) {
        // a thread's run is one label row of NSL consecutive slots, 32-byte aligned
        // when the outputs are: 32-byte stores, one sector each
        if (a.out_v8) {
          if (mvalid) {
#pragma unroll
            for (int c2 = 0; c2 < NSL / 16; ++c2) {
              if constexpr (kUpd == 0) {
                st_global_bf16x16(a.dW + o + 16 * c2, &v[16 * c2]);
              } else {
                float mo[16], wo[16];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(&wv[2 * c2 + h]);
                  const __nv_bfloat16* mb = reinterpret_cast<const __nv_bfloat16*>(&mv[2 * c2 + h]);
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const float d = v[16 * c2 + 8 * h + e];
                    mo[8 * h + e] = kUpd == 2 ? fmaf(a.momentum, __bfloat162float(mb[e]), d) : d;
                    wo[8 * h + e] = fmaf(-a.lr, mo[8 * h + e], __bfloat162float(wb[e]));
                  }
                }
                if constexpr (kUpd == 2) st_global_bf16x16(a.M + o + 16 * c2, mo);
                st_global_bf16x16(a.W_out + o + 16 * c2, wo);
              }
            }
          }
          stored = true;
        }
      }
      if (!stored && mvalid) {
#pragma unroll
        for (int c = 0; c < NSL / 8; ++c) {
          float d8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) d8[e] = v[8 * c + e];
          if constexpr (kUpd == 0) {
            *reinterpret_cast<uint4*>(a.dW + o + 8 * c) =
                make_uint4(pack_bf16x2(d8[0], d8[1]), pack_bf16x2(d8[2], d8[3]), pack_bf16x2(d8[4], d8[5]),
                           pack_bf16x2(d8[6], d8[7]));
          } else {
            const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(&wv[c]);
            const __nv_bfloat16* mb = reinterpret_cast<const __nv_bfloat16*>(&mv[c]);
            float mo[8], wo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              mo[e] = kUpd == 2 ? fmaf(a.momentum, __bfloat162float(mb[e]), d8[e]) : d8[e];
              wo[e] = fmaf(-a.lr, mo[e], __bfloat162float(wb[e]));
            }
            if constexpr (kUpd == 2)
              *reinterpret_cast<uint4*>(a.M + o + 8 * c) =
                  make_uint4(pack_bf16x2(mo[0], mo[1]), pack_bf16x2(mo[2], mo[3]), pack_bf16x2(mo[4], mo[5]),
                             pack_bf16x2(mo[6], mo[7]));
            *reinterpret_cast<uint4*>(a.W_out + o + 8 * c) =
                make_uint4(pack_bf16x2(wo[0], wo[1]), pack_bf16x2(wo[2], wo[3]), pack_bf16x2(wo[4], wo[5]),
                           pack_bf16x2(wo[6], wo[7]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[s]);
      return true;
    };
    // iteration i: the BCE of group i, then the dW readout of group i - 1.  Every
    // epilogue thread passes the same named barriers: a readout that fails stops
    // the loop only at the next BCE's barrier.
    bool failed = false, all_bce = true;
    for (int i = 0; i <= n_items; ++i) {
      if (i < n_items && !bce(i, failed)) {
        all_bce = false;
        break;
      }
      if (i >= 1 && !failed) failed = !readout(i - 1);
    }
    // deterministic loss reduction over the epilogue warps (named barrier 1)
    float v = loss_acc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[ew] = v;
    named_bar(1, kStepEpiThreads);
    if (storer) {
      float t = 0.f;
      for (int j = 0; j < kStepEpi; ++j) t += red[j];
      a.loss_part[blockIdx.x] = t;
      if (all_bce && n_items > 0) store_dy(n_items - 1);  // every warp has written it (barrier above)
      bulk_wait_all();  // the CTA exits only once its stores are complete
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
  // the gradient buffer [n_items * 64][Bp] (label rows, items of 64 / G groups) as
  // the stores' tensor: group g's G label rows, one box per 64 batch columns
  CUtensorMap tm_dy;
  const uint64_t n_items = (uint64_t)(a.sh.n_groups + 64 / kG - 1) / (64 / kG);
  e = tmap_2d(&tm_dy, a.dY_out, (uint64_t)a.sh.Bp, n_items * 64, (uint64_t)a.sh.Bp * 2, 64, kG);
  if (e != cudaSuccess) return e;
  kern<<<grid, v2::step_threads(v2::step_wide(kG, kUpd)), smem, st>>>(a, static_cast<const __nv_bfloat16*>(Xt),
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
