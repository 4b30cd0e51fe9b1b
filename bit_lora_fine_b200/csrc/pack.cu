// Packs the low-rank factors into the K-major layouts the tensor-core kernels
// read, and clears the per-call bookkeeping (status word, split counters).
//
// With D = [S_dn | A] ([K, R], R = r_s + r) and U = [S_up ; B] ([R, N]):
//   forward  needs D^T [R, K] (B operand of X*D) and U^T [N, R] (B operand of L*U)
//   backward needs U   [R, N] (B operand of G*U^T) and D   [K, R] (B operand of P*D^T)
#include "common.cuh"
#include "kernels.h"

namespace ft {

__global__ void pack_lowrank_kernel(PackParams p) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  const int R = p.r_s + p.r;
  // bookkeeping first: status word and split counters start at zero every call
  for (long long i = tid; i < p.n_zero_words; i += nthreads) p.zero_words[i] = 0;
  const uint16_t* Sdn = static_cast<const uint16_t*>(p.S_dn);
  const uint16_t* A = static_cast<const uint16_t*>(p.A);
  const uint16_t* Sup = static_cast<const uint16_t*>(p.S_up);
  const uint16_t* B = static_cast<const uint16_t*>(p.B);
  if (p.Dt) {  // Dt[j, k]
    for (long long i = tid; i < static_cast<long long>(R) * p.K; i += nthreads) {
      const int j = static_cast<int>(i / p.K), k = static_cast<int>(i % p.K);
      p.Dt[i] = j < p.r_s ? Sdn[static_cast<long long>(k) * p.r_s + j] : A[static_cast<long long>(k) * p.r + (j - p.r_s)];
    }
  }
  if (p.Dcat) {  // Dcat[k, j]
    for (long long i = tid; i < static_cast<long long>(R) * p.K; i += nthreads) {
      const int k = static_cast<int>(i / R), j = static_cast<int>(i % R);
      p.Dcat[i] = j < p.r_s ? Sdn[static_cast<long long>(k) * p.r_s + j] : A[static_cast<long long>(k) * p.r + (j - p.r_s)];
    }
  }
  if (p.Ut) {  // Ut[n, j]
    for (long long i = tid; i < static_cast<long long>(R) * p.N; i += nthreads) {
      const int n = static_cast<int>(i / R), j = static_cast<int>(i % R);
      p.Ut[i] = j < p.r_s ? Sup[static_cast<long long>(j) * p.N + n] : B[static_cast<long long>(j - p.r_s) * p.N + n];
    }
  }
  if (p.Ucat) {  // Ucat[j, n]
    for (long long i = tid; i < static_cast<long long>(R) * p.N; i += nthreads) {
      const int j = static_cast<int>(i / p.N), n = static_cast<int>(i % p.N);
      p.Ucat[i] = j < p.r_s ? Sup[static_cast<long long>(j) * p.N + n] : B[static_cast<long long>(j - p.r_s) * p.N + n];
    }
  }
}

cudaError_t launch_pack_lowrank(const PackParams& p, int num_sms, cudaStream_t stream) {
  pack_lowrank_kernel<<<num_sms * 2, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ft
