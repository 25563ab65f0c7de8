// roles.cu -- head roles from HardKuma gate parameters.
//
// Page "LycheeDecode: Accelerating Long-Context LLM Inference via Hybrid-Head
// Sparse Decoding" (paper.rainbus.top/paper/2602.04541): the gate of head h in
// layer l is z ~ HardKuma(alpha, beta) (method step (2)); at inference the head
// is a retrieval head when E[z] > 0.5 (step (7)), and the expected L0 norm of
// the gates is sum over heads of 1 - F(-p / (q - p); alpha, beta) with F the
// Kumaraswamy CDF (the novelty paragraph).  Layer 0 is all retrieval (step (1)).
//
// HardKuma: K ~ Kumaraswamy(alpha, beta) on (0, 1), F(x) = 1 - (1 - x^alpha)^beta,
// stretched to T = p + (q - p) K (p < 0 < 1 < q) and rectified to
// z = min(1, max(0, T)).  z is a non-decreasing function g of K with g(0) = 0
// and slope q - p on (a, b), a = -p / (q - p), b = (1 - p) / (q - p), flat
// elsewhere, so integrating by parts
//     E[z] = integral_0^1 g'(k) P(K > k) dk = (q - p) integral_a^b (1 - k^alpha)^beta dk,
// an integral of a smooth function bounded by 1 over an interval inside (0, 1).
// It is evaluated here by composite Simpson's rule with kPanels panels, in
// fp64.  P(z != 0) = 1 - F(a) = (1 - a^alpha)^beta.
//
// One CTA; thread t takes heads t, t + kThreads, ...; the expected L0 norm is
// summed per thread in head order and then over threads in a fixed tree, so
// the result does not depend on scheduling.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace lychee {
namespace {

constexpr int kThreads = 1024;
constexpr int kPanels = 2048;   // Simpson panels (even) over [a, b]

// P(K > x) = (1 - x^alpha)^beta for x in (0, 1), through logarithms so that
// small x^alpha keeps its precision.
__device__ __forceinline__ double kuma_survival(double x, double alpha, double beta) {
  const double u = exp(alpha * log(x));
  return exp(beta * log1p(-u));
}

__global__ void __launch_bounds__(kThreads) hardkuma_roles_kernel(const __grid_constant__ RolesParams p) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ double red[kThreads];
  const int n = p.L * p.Hq;
  const double a = -p.p / (p.q - p.p), b = (1.0 - p.p) / (p.q - p.p);
  const double hs = (b - a) / kPanels;
  double l0 = 0.0;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const double alpha = p.alpha[i], beta = p.beta[i];
    double ez = NAN, nz = NAN;
    if (alpha > 0.0 && beta > 0.0 && alpha < INFINITY && beta < INFINITY) {
      double s_odd = 0.0, s_even = 0.0;
      for (int j = 1; j < kPanels; j += 2) s_odd += kuma_survival(a + j * hs, alpha, beta);
      for (int j = 2; j < kPanels; j += 2) s_even += kuma_survival(a + j * hs, alpha, beta);
      const double fa = kuma_survival(a, alpha, beta), fb = kuma_survival(b, alpha, beta);
      ez = (p.q - p.p) * (hs / 3.0) * (fa + fb + 4.0 * s_odd + 2.0 * s_even);
      nz = fa;
    }
    const bool layer0 = p.layer0_retrieval && i < p.Hq;
    p.role[i] = (layer0 || ez > 0.5) ? 1 : 0;   // NaN (bad parameters): sparse
    if (p.expected_z) p.expected_z[i] = ez;
    if (!layer0) l0 += nz;
  }
  red[threadIdx.x] = l0;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0 && p.expected_l0) *p.expected_l0 = red[0];
}

}  // namespace

cudaError_t launch_hardkuma_roles(const RolesParams& p, cudaStream_t st) {
  const cudaError_t e = launch_pdl(hardkuma_roles_kernel, dim3(1), dim3(kThreads), 0, st, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lychee
