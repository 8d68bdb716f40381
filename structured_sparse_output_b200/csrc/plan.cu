// plan.cu -- the plan's inverse map built on the device (HASTE, "Hardware-Aware
// Dynamic Sparse Training for Large Output Spaces": Methodology 1 stores one
// index set I_g per group; the title's dynamic sparse training rewires those sets
// during training, and every rewiring needs the map feature -> (group, slot)
// again).
//
// A stable counting sort of the entries e = g*k + s by feature idx[e], on the
// device, in three passes over group chunks (chunk c = groups
// [c*n/C, (c+1)*n/C)):
//   k_plan_hist     per chunk, the count of each feature (shared-memory integer
//                   counters: exact in any order);
//   k_plan_prefix   per feature, the exclusive prefix of its counts over the
//                   chunks (cnt[c][f] becomes the number of entries of feature f
//                   in chunks before c) and its total;
//   k_plan_scan     the exclusive prefix of the totals over the features: inv_off;
//   k_plan_scatter  per chunk, its groups in ascending order: the thread of slot
//                   s places e = g*k + s at the running position of feature
//                   idx[g, s] (a group's features are distinct, so no two threads
//                   of one step share a counter).
// Entries of one feature therefore land in ascending group order: the same
// arrays as the host construction, bit for bit.
// k_plan_set_rows writes replaced index rows into the plan's idx array.

#include "common.cuh"

namespace haste {
namespace plan {

constexpr int kMaxChunks = 1024;
constexpr int kThreads = 256;

__host__ __device__ inline int64_t chunk_begin(int c, int64_t n_groups, int n_chunks) {
  return (int64_t)c * n_groups / n_chunks;
}

__global__ void __launch_bounds__(kThreads) k_plan_hist(const int32_t* __restrict__ idx, int64_t n_groups, int k,
                                                         int d, int n_chunks, int32_t* __restrict__ cnt) {
  extern __shared__ int32_t h[];
  for (int f = threadIdx.x; f < d; f += blockDim.x) h[f] = 0;
  __syncthreads();
  const int c = blockIdx.x;
  const int64_t e0 = chunk_begin(c, n_groups, n_chunks) * k, e1 = chunk_begin(c + 1, n_groups, n_chunks) * k;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) atomicAdd(&h[idx[e]], 1);
  __syncthreads();
  for (int f = threadIdx.x; f < d; f += blockDim.x) cnt[(int64_t)c * d + f] = h[f];
}

__global__ void __launch_bounds__(kThreads) k_plan_prefix(int32_t* __restrict__ cnt, int d, int n_chunks,
                                                           int32_t* __restrict__ tot) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= d) return;
  int32_t run = 0;
  for (int c = 0; c < n_chunks; ++c) {
    const int32_t t = cnt[(int64_t)c * d + f];
    cnt[(int64_t)c * d + f] = run;
    run += t;
  }
  tot[f] = run;
}

// One block: inv_off[f] = sum of tot[0..f), inv_off[d] = the total.  Thread i
// covers the consecutive features [i*per, (i+1)*per).
__global__ void __launch_bounds__(1024) k_plan_scan(const int32_t* __restrict__ tot, int d,
                                                     int32_t* __restrict__ inv_off) {
  __shared__ int32_t part[1024];
  const int per = (d + blockDim.x - 1) / blockDim.x;
  const int f0 = threadIdx.x * per, f1 = min(d, f0 + per);
  int32_t s = 0;
  for (int f = f0; f < f1; ++f) s += tot[f];
  part[threadIdx.x] = s;
  __syncthreads();
  // inclusive scan of the per-thread sums (Hillis-Steele; integers, exact)
  for (int o = 1; o < (int)blockDim.x; o <<= 1) {
    const int32_t v = threadIdx.x >= (unsigned)o ? part[threadIdx.x - o] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int32_t run = part[threadIdx.x] - s;
  for (int f = f0; f < f1; ++f) {
    inv_off[f] = run;
    run += tot[f];
  }
  if (threadIdx.x == blockDim.x - 1) inv_off[d] = part[threadIdx.x];
}

__global__ void __launch_bounds__(kThreads) k_plan_scatter(const int32_t* __restrict__ idx, int64_t n_groups, int k,
                                                            int d, int n_chunks, const int32_t* __restrict__ cnt,
                                                            const int32_t* __restrict__ inv_off,
                                                            int32_t* __restrict__ inv_ent) {
  extern __shared__ int32_t pos[];
  const int c = blockIdx.x;
  for (int f = threadIdx.x; f < d; f += blockDim.x) pos[f] = inv_off[f] + cnt[(int64_t)c * d + f];
  __syncthreads();
  const int64_t g0 = chunk_begin(c, n_groups, n_chunks), g1 = chunk_begin(c + 1, n_groups, n_chunks);
  // groups in ascending order; kThreads / k groups' rows per step would reorder
  // equal features, so one group per step
  for (int64_t g = g0; g < g1; ++g) {
    for (int s = threadIdx.x; s < k; s += blockDim.x) {
      const int32_t f = idx[g * k + s];
      const int32_t p = pos[f];
      pos[f] = p + 1;
      inv_ent[p] = (int32_t)(g * k + s);
    }
    __syncthreads();
  }
}

// rows [n_changed][k] replace the index rows of groups[0..n_changed)
__global__ void k_plan_set_rows(int32_t* __restrict__ idx, int k, const int32_t* __restrict__ groups,
                                const int32_t* __restrict__ rows, int64_t n_changed) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_changed * k) return;
  const int64_t r = i / k;
  idx[(int64_t)groups[r] * k + (i % k)] = rows[i];
}

// Scratch of the device build: int32 counts [n_chunks][d] and totals [d].
inline int n_chunks_for(int64_t n_groups) { return (int)std::min<int64_t>(n_groups, kMaxChunks); }
inline size_t scratch_ints(int64_t n_groups, int d) { return (size_t)n_chunks_for(n_groups) * d + d; }

// The inverse map of the device index array idx [n_groups, k] (validated), with
// scratch of scratch_ints() ints.  Needs d * 4 bytes of shared memory per block.
cudaError_t build_inverse(const int32_t* idx, int64_t n_groups, int k, int d, int32_t* scratch, int32_t* inv_off,
                          int32_t* inv_ent, cudaStream_t st) {
  const int C = n_chunks_for(n_groups);
  int32_t* cnt = scratch;
  int32_t* tot = scratch + (size_t)C * d;
  const size_t smem = (size_t)d * 4;
  cudaError_t e = cudaSuccess;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(k_plan_hist, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_plan_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_plan_hist<<<C, kThreads, smem, st>>>(idx, n_groups, k, d, C, cnt);
  k_plan_prefix<<<(d + kThreads - 1) / kThreads, kThreads, 0, st>>>(cnt, d, C, tot);
  k_plan_scan<<<1, 1024, 0, st>>>(tot, d, inv_off);
  k_plan_scatter<<<C, k <= 128 ? 128 : kThreads, smem, st>>>(idx, n_groups, k, d, C, cnt, inv_off, inv_ent);
  return cudaGetLastError();
}

}  // namespace plan
}  // namespace haste
