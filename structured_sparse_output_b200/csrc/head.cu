// head.cu -- the dense head classifier on the 5th-gen tensor cores.
//
// HASTE ("Hardware-Aware Dynamic Sparse Training for Large Output Spaces"),
// Methodology 2 "Head-Tail Decomposition": the few frequent labels are modelled by
// a standard dense classifier next to the group-shared sparse tail.
//   forward : logits_h = Xh . Wh^T               (M = batch, N = H, K = d)
//   dWh     : dWh = dY_h^T . Xh                   (M = H, N = d, K = batch)
//   dXh     : dXh = dY_h . Wh                     (M = batch, N = d, K = H)
// One tcgen05 GEMM kernel D[M,N] = A[M,K] . B[N,K]^T covers the three products;
// each operand is read from global memory either K-contiguous or MN-contiguous
// and staged into the matching 128B-swizzled canonical layout.
#include "common.cuh"

namespace haste {
namespace {

constexpr int kGThreads = 128;
constexpr int kBM = 128;
constexpr int kFwdN = 64;  // output tile width of the forward (B x H has few 128-wide tiles)

enum Epi : int { kEpiStore = 0, kEpiStoreF32 = 1, kEpiPartial = 2, kEpiBce = 3 };

struct GemmArgs {
  const void* A;   // element (m, k) at A[m*lda + k] (K-major) or A[k*lda + m] (MN-major)
  const void* Bm;  // element (n, k) at B[n*ldb + k] (K-major) or B[k*ldb + n] (MN-major)
  int64_t lda, ldb;
  int M, N, K;
  int k_per_split;
  void* C;          // output [M, N] row-major (ldc), or partials [splits, M, N] fp32
  int64_t ldc;
  // BCE epilogue
  const int32_t* pos_ptr;
  const int32_t* pos_ids;
  float scale;
  float* loss_part;
};

// Stage a kRows x BK tile of an operand whose rows are the M (or N) index
// (kRows = 128, or 64 for a K-major operand).
template <typename T, bool kMN, int kRows = 128>
__device__ __forceinline__ void load_operand(uint32_t s, const T* __restrict__ p, int64_t ld, int rows, int K,
                                             int r0, int k0, int BK) {
  constexpr int CW = 16 / sizeof(T);
  static_assert(kRows == 128 || (kRows == 64 && !kMN), "64-row tiles are K-major only");
  if constexpr (!kMN) {
    // K-major: [k-block][row][128B]
    const int cpr = BK / CW;
    for (int i = threadIdx.x; i < kRows * cpr; i += blockDim.x) {
      const int r = i / cpr, cc = i % cpr;
      const int gr = r0 + r, gk = k0 + cc * CW;
      const bool in = gr < rows && gk < K;
      const T* src = in ? p + (int64_t)gr * ld + gk : p;
      const uint32_t off = (uint32_t)((cc >> 3) * kRows * 128 + r * 128 + (cc & 7) * 16);
      cp_async16(s + sw128(off), src, in ? 16u : 0u);
    }
  } else {
    // MN-major: [row-block of R][k][128B]
    const int cpr = 128 / CW;
    for (int i = threadIdx.x; i < BK * cpr; i += blockDim.x) {
      const int kr = i / cpr, cc = i % cpr;
      const int gk = k0 + kr, gr = r0 + cc * CW;
      const bool in = gk < K && gr < rows;
      const T* src = in ? p + (int64_t)gk * ld + gr : p;
      const uint32_t off = (uint32_t)((cc >> 3) * BK * 128 + kr * 128 + (cc & 7) * 16);
      cp_async16(s + swz<T, true>(off), src, in ? 16u : 0u);
    }
  }
}

template <typename T, bool kMN, int kRows = 128>
__device__ __forceinline__ uint64_t operand_desc(uint32_t s, int kk, int BK) {
  constexpr int R = 128 / sizeof(T), KI = Elem<T>::kMmaK;
  if constexpr (!kMN) {
    return make_sdesc(s + (uint32_t)(((kk * KI) / R) * kRows * 128 + (kk % (R / KI)) * 32), 16, 1024,
                      kLayoutSw128);
  } else {
    return mn_desc<T>(s + (uint32_t)(kk * KI * 128), (uint32_t)BK * 128);
  }
}

template <typename T, bool kAMN, bool kBMN, int kEpi, int kBN, int kStages>
__global__ void __launch_bounds__(kGThreads, 1) k_gemm(GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int R = 128 / sizeof(T), KI = Elem<T>::kMmaK;
  constexpr int BK = 2 * R;  // two 128B rows of K per stage
  // kStages = 2: the operands of K chunk i+1 load while the MMAs of chunk i run
  // (for grids that leave SMs idle); kStages = 1: several CTAs share an SM and
  // overlap each other
  constexpr uint32_t kStageA = (uint32_t)kBM * BK * sizeof(T), kStageB = (uint32_t)kBN * BK * sizeof(T);
  const uint32_t base = align1024(smem_u32(smem));
  auto SA = [&](int st) -> uint32_t { return base + (uint32_t)st * (kStageA + kStageB); };
  auto SB = [&](int st) -> uint32_t { return SA(st) + kStageA; };
  uint8_t* gen = smem + (base + kStages * (kStageA + kStageB) - smem_u32(smem));
  uint64_t* bar = reinterpret_cast<uint64_t*>(gen);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  float* red = reinterpret_cast<float*>(abort_flag + 1);

  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN, split = blockIdx.z;
  const int k_begin = split * a.k_per_split;
  const int k_end = min(a.K, k_begin + a.k_per_split);

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(tslot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  uint32_t phase = 0;
  const uint32_t idesc = make_idesc(Elem<T>::kFmt, kAMN ? 1u : 0u, kBMN ? 1u : 0u, 128, kBN);
  const T* A = static_cast<const T*>(a.A);
  const T* Bm = static_cast<const T*>(a.Bm);
  bool ok = true;

  auto load = [&](int k0, int st) {
    load_operand<T, kAMN>(SA(st), A, a.lda, a.M, k_end, m0, k0, BK);
    load_operand<T, kBMN, kBN>(SB(st), Bm, a.ldb, a.N, k_end, n0, k0, BK);
    cp_async_commit();
  };
  const int n_chunks = k_end > k_begin ? (k_end - k_begin + BK - 1) / BK : 0;
  if (kStages == 2 && n_chunks > 0) load(k_begin, 0);
  for (int it = 0; it < n_chunks; ++it) {
    const int st = kStages == 2 ? (it & 1) : 0;
    if constexpr (kStages == 1) {
      // the stage was read by the MMAs of chunk it-1
      if (it >= 1) {
        const bool w = mbar_wait(bar, phase);
        phase ^= 1u;
        if (!w) *abort_flag = 1;
      }
      load(k_begin + it * BK, 0);
      cp_async_wait_all();
    } else if (it + 1 < n_chunks) {
      // the other stage was read by the MMAs of chunk it-1: wait for them, then load chunk it+1 into it
      if (it >= 1) {
        const bool w = mbar_wait(bar, phase);
        phase ^= 1u;
        if (!w) *abort_flag = 1;
      }
      load(k_begin + (it + 1) * BK, st ^ 1);
      cp_async_wait_group<1>();  // chunk it has landed
    } else {
      if (it >= 1) {
        const bool w = mbar_wait(bar, phase);
        phase ^= 1u;
        if (!w) *abort_flag = 1;
      }
      cp_async_wait_all();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) {
      ok = false;
      break;
    }
    if (threadIdx.x == 0) {
      const uint32_t sa = SA(st), sb = SB(st);
      for (int kk = 0; kk < BK / KI; ++kk)
        mma_ss<Elem<T>::kTF32>(tmem, operand_desc<T, kAMN>(sa, kk, BK), operand_desc<T, kBMN, kBN>(sb, kk, BK), idesc,
                               (it > 0 || kk > 0) ? 1u : 0u);
      mma_commit(bar);
    }
  }
  // the MMAs of the last chunk
  if (ok && n_chunks > 0) {
    const bool w = mbar_wait(bar, phase);
    phase ^= 1u;
    if (!w) *abort_flag = 1;
    tc_fence_after();
    __syncthreads();
    if (*abort_flag) ok = false;
  }
  cp_async_wait_all();

  const int m = m0 + threadIdx.x;
  const uint32_t lane = tmem + (((threadIdx.x / 32) * 32u) << 16);
  float loss_acc = 0.f;
  if (ok && k_end > k_begin) {
    uint64_t ym0 = 0, ym1 = 0;
    if constexpr (kEpi == kEpiBce) {
      if (m < a.M)
        for (int p = a.pos_ptr[m]; p < a.pos_ptr[m + 1]; ++p) {
          const int l = a.pos_ids[p] - n0;
          if (l >= 0 && l < 64) ym0 |= 1ull << l;
          else if (l >= 64 && l < kBN) ym1 |= 1ull << (l - 64);
        }
    }
    for (int c = 0; c < kBN; c += 16) {
      float v[16];
      tmem_ld16(lane + (uint32_t)c, v);
      tmem_wait_ld();
      if (m >= a.M) continue;
      const int n = n0 + c;
      if constexpr (kEpi == kEpiPartial || kEpi == kEpiStoreF32) {
        float* dst = kEpi == kEpiPartial ? static_cast<float*>(a.C) + ((int64_t)split * a.M + m) * a.N + n
                                         : static_cast<float*>(a.C) + (int64_t)m * a.ldc + n;
        const int64_t ld = kEpi == kEpiPartial ? a.N : a.ldc;
        if (n + 16 <= a.N && (ld & 3) == 0 && (reinterpret_cast<uintptr_t>(a.C) & 15) == 0) {  // 4 x 16 B
#pragma unroll
          for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        } else {
          for (int i = 0; i < 16; ++i)
            if (n + i < a.N) dst[i] = v[i];
        }
      } else {
        if constexpr (kEpi == kEpiBce) {
          float lin = 0.f, prod = 1.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int j = c + i;
            const uint64_t mk = j < 64 ? ym0 : ym1;
            const float y = ((mk >> (j & 63)) & 1ull) ? 1.f : 0.f;
            const float th = tanh_approx(0.5f * v[i]);
            const bool in = n + i < a.N;
            lin += in ? fmaxf(v[i], 0.f) - v[i] * y : 0.f;
            prod *= in ? fmaf(0.5f, fabsf(th), 0.5f) : 1.f;
            v[i] = a.scale * (fmaf(0.5f, th, 0.5f) - y);
          }
          loss_acc += lin - __logf(prod);
        }
        T* dst = static_cast<T*>(a.C) + (int64_t)m * a.ldc + n;
        if (sizeof(T) == 2 && n + 16 <= a.N && (a.ldc & 7) == 0 &&
            (reinterpret_cast<uintptr_t>(a.C) & 15) == 0) {  // 2 x 16 B
#pragma unroll
          for (int i = 0; i < 16; i += 8)
            *reinterpret_cast<uint4*>(dst + i) =
                make_uint4(pack_bf16x2(v[i], v[i + 1]), pack_bf16x2(v[i + 2], v[i + 3]),
                           pack_bf16x2(v[i + 4], v[i + 5]), pack_bf16x2(v[i + 6], v[i + 7]));
        } else {
          for (int i = 0; i < 16; ++i)
            if (n + i < a.N) dst[i] = Elem<T>::from_f(v[i]);
        }
      }
    }
  }
  if constexpr (kEpi == kEpiBce) {
    float v = loss_acc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) a.loss_part[blockIdx.y * gridDim.x + blockIdx.x] = ((red[0] + red[1]) + red[2]) + red[3];
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// out[m, n] = sum over splits s ascending of P[s, m, n]
__global__ void k_split_reduce(const float* __restrict__ P, float* __restrict__ out, int S, int64_t MN) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < MN; i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int sp = 0; sp < S; ++sp) s += P[sp * MN + i];
    out[i] = s;
  }
}

template <typename T, bool kAMN, bool kBMN, int kEpi, int kBN, int kStages>
cudaError_t run_gemm_t(const GemmArgs& a, dim3 grid, cudaStream_t st) {
  constexpr int BK = 2 * (128 / (int)sizeof(T));
  const size_t smem = 1024 + kStages * (size_t)(kBM + kBN) * BK * sizeof(T) + 64;
  auto kern = k_gemm<T, kAMN, kBMN, kEpi, kBN, kStages>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kGThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// Two stages when the grid leaves SMs without a CTA, one (several CTAs per SM)
// otherwise.
template <typename T, bool kAMN, bool kBMN, int kEpi, int kBN = 128>
cudaError_t run_gemm(const GemmArgs& a, int splits, cudaStream_t st) {
  const dim3 grid((a.M + kBM - 1) / kBM, (a.N + kBN - 1) / kBN, splits);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 0;
  if ((int64_t)grid.x * grid.y * grid.z <= sms) return run_gemm_t<T, kAMN, kBMN, kEpi, kBN, 2>(a, grid, st);
  return run_gemm_t<T, kAMN, kBMN, kEpi, kBN, 1>(a, grid, st);
}

}  // namespace

namespace head {

// Work split of dXh (K = H can be long): K chunks of a multiple of the stage depth,
// about 512 long, so that the few output tiles (B/128 x d/128) still fill the SMs.
int dxh_splits(int H, int elem) {
  const int BK = 2 * (128 / elem);
  int s = H / 512;
  if (s < 1) s = 1;
  if (s > 32) s = 32;
  while (s > 1 && ((H + s - 1) / s) % BK) --s;
  return s;
}

int fwd_tiles(int B, int H) { return ((B + kBM - 1) / kBM) * ((H + kFwdN - 1) / kFwdN); }

template <typename T>
cudaError_t forward(int B, int H, int d, const void* Xh, const void* Wh, void* out, const int32_t* pos_ptr,
                    const int32_t* pos_ids, float scale, float* loss_part, cudaStream_t st) {
  GemmArgs a{};
  a.A = Xh;
  a.lda = d;
  a.Bm = Wh;
  a.ldb = d;
  a.M = B;
  a.N = H;
  a.K = d;
  a.k_per_split = d;
  a.C = out;
  a.ldc = H;
  if (pos_ptr) {
    a.pos_ptr = pos_ptr;
    a.pos_ids = pos_ids;
    a.scale = scale;
    a.loss_part = loss_part;
    return run_gemm<T, false, false, kEpiBce, kFwdN>(a, 1, st);
  }
  return run_gemm<T, false, false, kEpiStore, kFwdN>(a, 1, st);
}

// dWh = dY_h^T . Xh : A(m=h, k=b) = dY_h[b, h] (MN-major), B(n=f, k=b) = Xh[b, f] (MN-major)
template <typename T>
cudaError_t backward_dw(int B, int H, int d, const void* Xh, const void* dYh, void* dWh, cudaStream_t st) {
  GemmArgs a{};
  a.A = dYh;
  a.lda = H;
  a.Bm = Xh;
  a.ldb = d;
  a.M = H;
  a.N = d;
  a.K = B;
  a.k_per_split = B;
  a.C = dWh;
  a.ldc = d;
  return run_gemm<T, true, true, kEpiStore>(a, 1, st);
}

// dXh = dY_h . Wh : A(m=b, k=h) = dY_h[b, h] (K-major), B(n=f, k=h) = Wh[h, f] (MN-major);
// split over K = H into fp32 partials reduced in a fixed order.
template <typename T>
cudaError_t backward_dx(int B, int H, int d, const void* Wh, const void* dYh, float* dXh, float* part,
                        cudaStream_t st) {
  const int S = dxh_splits(H, sizeof(T));
  GemmArgs a{};
  a.A = dYh;
  a.lda = H;
  a.Bm = Wh;
  a.ldb = d;
  a.M = B;
  a.N = d;
  a.K = H;
  a.k_per_split = (H + S - 1) / S;
  a.C = S > 1 ? (void*)part : (void*)dXh;
  a.ldc = d;
  if (S == 1) return run_gemm<T, false, true, kEpiStoreF32>(a, 1, st);
  cudaError_t e = run_gemm<T, false, true, kEpiPartial>(a, S, st);
  if (e != cudaSuccess) return e;
  const int64_t MN = (int64_t)B * d;
  k_split_reduce<<<(int)((MN + 255) / 256 < 1184 ? (MN + 255) / 256 : 1184), 256, 0, st>>>(part, dXh, S, MN);
  return cudaGetLastError();
}

template cudaError_t forward<float>(int, int, int, const void*, const void*, void*, const int32_t*, const int32_t*,
                                    float, float*, cudaStream_t);
template cudaError_t forward<__nv_bfloat16>(int, int, int, const void*, const void*, void*, const int32_t*,
                                            const int32_t*, float, float*, cudaStream_t);
template cudaError_t backward_dw<float>(int, int, int, const void*, const void*, void*, cudaStream_t);
template cudaError_t backward_dw<__nv_bfloat16>(int, int, int, const void*, const void*, void*, cudaStream_t);
template cudaError_t backward_dx<float>(int, int, int, const void*, const void*, float*, float*, cudaStream_t);
template cudaError_t backward_dx<__nv_bfloat16>(int, int, int, const void*, const void*, float*, float*,
                                                cudaStream_t);

}  // namespace head
}  // namespace haste
