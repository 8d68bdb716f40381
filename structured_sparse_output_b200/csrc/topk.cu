// topk.cu -- two-stage top-K scoring of the group-shared sparse tail on sm_100a.
//
// Scores: the logits of the HASTE tail ("HASTE: Hardware-Aware Dynamic Sparse
// Training for Large Output Spaces", Methodology 1), logits_g = X[:, I_g] . W_g^T.
// Selection: the two-stage approximate top-K of "A Faster Generalized Two-Stage
// Approximate Top-K" (Methodology): stage 1 keeps the top K' scores of each bucket,
// stage 2 the top K of the buckets' survivors; K' = K gives the exact top K.
// Buckets are contiguous runs of whole groups, one per CTA of stage 1, so the
// B x L logits are ranked inside the forward epilogue and never leave the chip.
// Rank order: larger logit first, equal logits by smaller label id.
//
// k_topk  -- stage 1, fused with the gather-once forward:
//   warps 0-3  cp.async producers (two per ring stage): the gathered tile
//              X[:, I_g] (k rows of X^T) and the G x k weight block;
//   warp 4     MMA issuer: logits of group i into TMEM F[i & 1];
//   warps 5-12 epilogue: warp (q, hh) keeps, for each batch row of its TMEM lane
//              quarter, the top K' of its half of every group's label columns
//              in registers; the two halves merge through shared memory at the end.
// k_topk_merge -- stage 2: one warp per sample picks the top K of the
//              n_buckets x K' candidates.
#include "tail.cuh"

namespace haste {
namespace topk {

constexpr int kThreads = 32 * (4 + 1 + 8);

struct Args {
  TailShape sh;
  const int32_t* idx;
  float* cand_val;  // [n_buckets][Bp][KP]
  int32_t* cand_id;
};

struct Layout {
  uint32_t xg[2], wg[2], xchg, bars, total;
};
__host__ __device__ inline Layout layout(int Bp, int k, int G, int KP) {
  Layout L;
  const uint32_t xg = (uint32_t)((Bp / 64) * k * 128 + (k < 128 ? (128 - k) * 128 : 0));
  const uint32_t wg = (uint32_t)((k / 64) * G * 128);
  uint32_t off = 0;
  for (int s = 0; s < 2; ++s) { L.xg[s] = off; off += xg; }
  for (int s = 0; s < 2; ++s) { L.wg[s] = off; off += wg; }
  L.xchg = off;  // [Bp][2 halves][KP] x (value, id)
  off += (uint32_t)(Bp * 2 * KP * 8);
  off = (off + 15) & ~15u;
  L.bars = off;
  off += 256;
  L.total = off + 1024;
  return L;
}

// (v1, i1) ranks before (v2, i2): larger value, then smaller id.
__device__ __forceinline__ bool ranks_before(float v1, int i1, float v2, int i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

// Insert (z, l) into the rank-ordered list (v, id) if it beats the last entry.
template <int KP>
__device__ __forceinline__ void keep_best(float (&v)[KP], int (&id)[KP], float z, int l) {
  if (!ranks_before(z, l, v[KP - 1], id[KP - 1])) return;
  v[KP - 1] = z;
  id[KP - 1] = l;
#pragma unroll
  for (int j = KP - 1; j > 0; --j) {
    if (ranks_before(v[j], id[j], v[j - 1], id[j - 1])) {
      const float tv = v[j];
      v[j] = v[j - 1];
      v[j - 1] = tv;
      const int ti = id[j];
      id[j] = id[j - 1];
      id[j - 1] = ti;
    }
  }
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity, g_wait_limit_ns)) {
    *abort_flag = 1;
    return false;
  }
  return true;
}

template <int kG, int kK, int KP>
__global__ void __launch_bounds__(kThreads, 1)
    k_topk(Args a, const __nv_bfloat16* __restrict__ Xt, const __nv_bfloat16* __restrict__ W) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int CH = kG / 2;  // label columns per epilogue half
  constexpr int kRows = kK / 8;  // index rows per producer lane
  const TailShape sh = a.sh;
  const int Bp = sh.Bp, n_bt = Bp / 128;
  const Layout Lo = layout(Bp, kK, kG, KP);
  const uint32_t base = align1024(smem_u32(smem));
  uint8_t* gbase = smem + (base - smem_u32(smem));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + Lo.bars);
  uint64_t* full = bars;          // [2] stage loaded (count: the stage's two producer warps)
  uint64_t* empty = bars + 2;     // [2] stage consumed by the forward product
  uint64_t* fwd_full = bars + 4;  // [2] logits in TMEM
  uint64_t* f_empty = bars + 6;   // [2] logits read out (count: 8 epilogue warps)
  uint64_t* done = bars + 8;      // every MMA of the CTA finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int w = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 64);
      mbar_init(&empty[s], 1);
      mbar_init(&fwd_full[s], 1);
      mbar_init(&f_empty[s], 8);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t f_cols = (uint32_t)(n_bt * kG);
  const uint32_t ncols = f_cols * 2 <= 32 ? 32 : f_cols * 2 <= 64 ? 64 : f_cols * 2 <= 128 ? 128 : 256;
  if (w == 4) {
    tmem_alloc(tslot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  auto F = [&](int s) -> uint32_t { return tmem + (s ? f_cols : 0u); };
  auto XG = [&](int s) -> uint32_t { return base + (s ? Lo.xg[1] : Lo.xg[0]); };
  auto WG = [&](int s) -> uint32_t { return base + (s ? Lo.wg[1] : Lo.wg[0]); };

  // this CTA's bucket: a contiguous run of groups
  const int64_t gb = (int64_t)blockIdx.x * sh.n_groups / gridDim.x;
  const int64_t ge = (int64_t)(blockIdx.x + 1) * sh.n_groups / gridDim.x;
  const int n_items = (int)(ge - gb);

  if (w < 4) {
    // ------------------------------------------------- cp.async producers
    // warps (half, part) fill stage half with the items i = half, half+2, ...;
    // lane (rg, sub) copies the 16-byte chunk sub of every 128-byte segment of
    // the rows rg + 4 (2m + part).
    const int half = w & 1, part = w >> 1;
    const int sub = lane & 7, rg = lane >> 3;
    const uint32_t xg = XG(half), wg = WG(half);
    for (int i = half; i < n_items; i += 2) {
      const int64_t g = gb + i;
      int idx_cur[kRows];
#pragma unroll
      for (int m = 0; m < kRows; ++m) idx_cur[m] = a.idx[g * kK + rg + 4 * (2 * m + part)];
      if (!wait_or_abort(&empty[half], ((i >> 1) & 1) ^ 1, abort_flag)) break;
      const int nbb = Bp / 64;
#pragma unroll
      for (int m = 0; m < kRows; ++m) {
        const int sl = rg + 4 * (2 * m + part);
        const __nv_bfloat16* src = Xt + (int64_t)idx_cur[m] * Bp + sub * 8;
        const uint32_t dst = xg + sw128((uint32_t)(sl * 128 + sub * 16));
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
          if (bb < nbb) cp_async16(dst + (uint32_t)(bb * kK * 128), src + bb * 64, 16);
      }
      const __nv_bfloat16* wsrc = W + g * (int64_t)kG * kK;
      constexpr int cpr = kK / 8;
#pragma unroll 4
      for (int c0 = 32 * part; c0 < kG * cpr; c0 += 64) {
        const int c = c0 + lane;
        const int j = c / cpr, cc = c % cpr;
        cp_async16(wg + sw128((uint32_t)((cc >> 3) * kG * 128 + j * 128 + (cc & 7) * 16)),
                   wsrc + (int64_t)j * kK + cc * 8, 16);
      }
      cp_async_commit();
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&full[half]);
    }
    cp_async_wait_all();
  } else if (w == 4) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = make_idesc(1, 1, 0, 128, kG);
    for (int i = 0; i < n_items; ++i) {
      const int s = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&f_empty[s], ((i >> 1) & 1) ^ 1, abort_flag))) break;
      if (!__all_sync(0xffffffffu, wait_or_abort(&full[s], (i >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      if (lane == 0) {
        for (int t = 0; t < n_bt; ++t)
          for (int kk = 0; kk < kK / 16; ++kk) {
            const uint64_t ad = make_sdesc(XG(s) + (uint32_t)(t * 2 * kK * 128 + kk * 16 * 128), (uint32_t)kK * 128,
                                           1024, kLayoutSw128);
            const uint64_t bd =
                make_sdesc(WG(s) + (uint32_t)((kk / 4) * kG * 128 + (kk % 4) * 32), 16, 1024, kLayoutSw128);
            mma_ss<false>(F(s) + (uint32_t)(t * kG), ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
        mma_commit(&fwd_full[s]);
        mma_commit(&empty[s]);
      }
      __syncwarp();
    }
    // also after an abort: TMEM is freed only once every issued MMA has finished
    if (lane == 0) mma_commit(done);
    __syncwarp();
    (void)__all_sync(0xffffffffu, mbar_wait(done, 0));
  } else {
    // ------------------------------------------------------------- epilogue
    // warp (q, hh): TMEM lane quarter q, label columns [hh*CH, hh*CH + CH)
    const int ew = w - 5, q = w & 3, hh = ew >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float v[2][KP];
    int id[2][KP];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int j = 0; j < KP; ++j) {
        v[t][j] = -INFINITY;
        id[t][j] = 0x7fffffff;
      }
    for (int i = 0; i < n_items; ++i) {
      const int s = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&fwd_full[s], (i >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const int l0 = (int)((gb + i) * kG + hh * CH);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= n_bt) break;
#pragma unroll
        for (int c = 0; c < CH; c += 16) {
          constexpr int NC = CH < 16 ? CH : 16;
          float z[16];
          if constexpr (NC == 8) tmem_ld8(F(s) + lane_off + (uint32_t)(t * kG + hh * CH + c), z);
          else tmem_ld16(F(s) + lane_off + (uint32_t)(t * kG + hh * CH + c), z);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < NC; ++e) keep_best<KP>(v[t], id[t], z[e], l0 + c + e);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&f_empty[s]);
    }
    // merge the two column halves of each batch row through shared memory
    float* xv = reinterpret_cast<float*>(gbase + Lo.xchg);
    int* xi = reinterpret_cast<int*>(xv + Bp * 2 * KP);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t >= n_bt) break;
      const int row = t * 128 + r;
#pragma unroll
      for (int j = 0; j < KP; ++j) {
        xv[(row * 2 + hh) * KP + j] = v[t][j];
        xi[(row * 2 + hh) * KP + j] = id[t][j];
      }
    }
    named_bar(1, 256);
    if (hh == 0) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= n_bt) break;
        const int row = t * 128 + r;
#pragma unroll
        for (int j = 0; j < KP; ++j) keep_best<KP>(v[t], id[t], xv[(row * 2 + 1) * KP + j], xi[(row * 2 + 1) * KP + j]);
        if (row < sh.B) {
#pragma unroll
          for (int j = 0; j < KP; ++j) {
            a.cand_val[((int64_t)blockIdx.x * Bp + row) * KP + j] = v[t][j];
            a.cand_id[((int64_t)blockIdx.x * Bp + row) * KP + j] = id[t][j];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// Stage 2: one warp per sample; K rounds of a warp-wide best-of over the
// n_buckets x KP candidates staged in shared memory.
__global__ void __launch_bounds__(32)
    k_topk_merge(const float* __restrict__ cand_val, const int32_t* __restrict__ cand_id, int Bp, int n_buckets,
                 int KP, int K, float* __restrict__ out_val, int32_t* __restrict__ out_id) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int b = blockIdx.x, lane = threadIdx.x;
  const int n = n_buckets * KP;
  float* sv = reinterpret_cast<float*>(smem);
  int* si = reinterpret_cast<int*>(sv + n);
  for (int c = lane; c < n; c += 32) {
    const int j = c / KP, e = c % KP;
    sv[c] = cand_val[((int64_t)j * Bp + b) * KP + e];
    si[c] = cand_id[((int64_t)j * Bp + b) * KP + e];
  }
  __syncwarp();
  for (int r = 0; r < K; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff, bc = -1;
    for (int c = lane; c < n; c += 32)
      if (ranks_before(sv[c], si[c], bv, bi)) {
        bv = sv[c];
        bi = si[c];
        bc = c;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      if (ranks_before(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
        bc = oc;
      }
    }
    if (lane == 0) {
      out_val[(int64_t)b * K + r] = bv;
      out_id[(int64_t)b * K + r] = bi;
      if (bc >= 0) {
        sv[bc] = -INFINITY;
        si[bc] = 0x7fffffff;
      }
    }
    __syncwarp();
  }
}

}  // namespace topk

// ------------------------------------------------------------- host side
namespace topk_host {

bool supported(int G, int k, int Bp, int kp) {
  return (G == 16 || G == 32 || G == 64) && (k == 64 || k == 128) && Bp <= 256 &&
         (kp == 1 || kp == 2 || kp == 4 || kp == 8);
}
size_t smem_stage1(int Bp, int k, int G, int kp) { return topk::layout(Bp, k, G, kp).total; }

template <int kG, int kK, int KP>
cudaError_t launch_t(const topk::Args& a, int grid, const void* Xt, const void* W, cudaStream_t st) {
  const size_t smem = smem_stage1(a.sh.Bp, kK, kG, KP);
  auto kern = topk::k_topk<kG, kK, KP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, topk::kThreads, smem, st>>>(a, static_cast<const __nv_bfloat16*>(Xt),
                                           static_cast<const __nv_bfloat16*>(W));
  return cudaGetLastError();
}

template <int kG, int kK>
cudaError_t launch_kp(int kp, const topk::Args& a, int grid, const void* Xt, const void* W, cudaStream_t st) {
  switch (kp) {
    case 1: return launch_t<kG, kK, 1>(a, grid, Xt, W, st);
    case 2: return launch_t<kG, kK, 2>(a, grid, Xt, W, st);
    case 4: return launch_t<kG, kK, 4>(a, grid, Xt, W, st);
    case 8: return launch_t<kG, kK, 8>(a, grid, Xt, W, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_stage1(int G, int k, int kp, const topk::Args& a, int grid, const void* Xt, const void* W,
                          cudaStream_t st) {
  switch (G * 1000 + k) {
    case 16064: return launch_kp<16, 64>(kp, a, grid, Xt, W, st);
    case 16128: return launch_kp<16, 128>(kp, a, grid, Xt, W, st);
    case 32064: return launch_kp<32, 64>(kp, a, grid, Xt, W, st);
    case 32128: return launch_kp<32, 128>(kp, a, grid, Xt, W, st);
    case 64064: return launch_kp<64, 64>(kp, a, grid, Xt, W, st);
    case 64128: return launch_kp<64, 128>(kp, a, grid, Xt, W, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_stage2(const float* cv, const int32_t* ci, int B, int Bp, int n_buckets, int kp, int K,
                          float* out_val, int32_t* out_id, cudaStream_t st) {
  const size_t smem = (size_t)n_buckets * kp * 8;
  cudaError_t e = cudaFuncSetAttribute(topk::k_topk_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk::k_topk_merge<<<B, 32, smem, st>>>(cv, ci, Bp, n_buckets, kp, K, out_val, out_id);
  return cudaGetLastError();
}

}  // namespace topk_host
}  // namespace haste
