// combine.cu -- merge of split partials into the attention output (method steps
// (3)/(4) of the page "LycheeDecode: Accelerating Long-Context LLM Inference via
// Hybrid-Head Sparse Decoding", paper.rainbus.top/paper/2602.04541).
//
// Chunk c of head h holds part_n[c] partial states (one per attention warp that
// served the head), each (m, l, a[d]) over a disjoint subset of the head's rows:
// m a reference raw dot, l = sum_j exp((s_j - m)/sqrt(d)) and a = sum_j exp(...)
// V_j.  With M = max m over all states and w = exp((m - M)/sqrt(d)):
// O = sum w a / sum w l, which is softmax(q K^T / sqrt(d)) V over the head's rows.
//
// kCombineSplit CTAs of 512 threads per (sequence, head), each over a range of
// the head's chunks.  Each lane owns four of the d elements of one "slot"; the
// range's states are listed in order and each slot takes every NS-th one,
// loading kBatch states before merging them into its running sums (rescaled
// when the maximum grows), so that the slot's loads are in flight together.
// The slots are merged in a fixed order in shared memory into one state per
// CTA.  The head's CTAs form one group of a thread-block cluster: each sends its
// state into the shared memory of the group's first CTA (16-byte st.async
// stores that complete that CTA's mbarrier), which merges the kCombineSplit
// states in order and writes the output.  The result does not depend on
// scheduling.
#include "combine_body.cuh"

namespace lychee {
namespace {

template <typename T, int D>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(const __grid_constant__ CombineParams p) {
  extern __shared__ __align__(16) unsigned char csm[];
  pdl_launch_dependents();
  combine_prologue<D>(csm);
  pdl_wait();
  combine_body<T, D>(p, blockIdx.x, csm);
}

template <typename T, int D>
cudaError_t launch_combine_t(const CombineParams& p, cudaStream_t st) {
  // clusters of kCombineSplit CTAs (a portable size): one head per cluster
  const unsigned grid = (unsigned)(p.B * p.Hq * kCombineSplit);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kCombThreads);
  cfg.dynamicSmemBytes = combine_smem_bytes<D>();
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kCombineSplit;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel<T, D>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int dtype, int D, cudaStream_t st) {
  if (dtype == 0 && D == 128) return launch_combine_t<__nv_bfloat16, 128>(p, st);
  if (dtype == 0 && D == 64) return launch_combine_t<__nv_bfloat16, 64>(p, st);
  if (dtype == 1 && D == 128) return launch_combine_t<float, 128>(p, st);
  if (dtype == 1 && D == 64) return launch_combine_t<float, 64>(p, st);
  return cudaErrorInvalidValue;
}

}  // namespace lychee
