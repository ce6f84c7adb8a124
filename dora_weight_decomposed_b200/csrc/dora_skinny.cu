// Token-contraction GEMMs of a low-rank layer, out[i][j] = sum_t P[t][i] Q[t][j]
// with i over a wide dimension (d_out or d_in) and j over a small rank
// (r <= 32): dB = dz^T su and dA^T = x^T du in the backward (DoRA notes eq. (7)
// through V' = W0 + s B A). At such ranks the contraction does 2r flops per
// element of the wide operand P, far below the tensor cores' ridge: it is a
// stream of P through HBM, so it runs on CUDA cores with every SM reading its
// own slice of P exactly once.
//
// Block: 64 columns of P x 256 tokens. Thread (column c, token group g) sums
// P[t][c] Q[t][0..R) over the tokens t = g, g + 4, ... of the block; the
// block's Q rows are staged in shared memory as fp32 (every thread of a group
// reads the same row: broadcast). The four token groups are added in shared
// memory in a fixed order and the block writes fp32 partials
// part[token block][i][j], which the split reduction sums in block order.
#include <algorithm>

#include <cuda_bf16.h>

#include "dora_internal.h"

namespace dora {
namespace {

constexpr int kSkCols = 64;     // columns of P per block
constexpr int kSkTokens = 256;  // tokens per block
constexpr int kSkGroups = 4;    // token groups (256 threads = 64 columns x 4 groups)

template <int R>
__global__ void __launch_bounds__(256) skinny_tn_kernel(const __nv_bfloat16* __restrict__ P, int ldp,
                                                        const __nv_bfloat16* __restrict__ Q, int ldq, int T, int W,
                                                        int r, float* __restrict__ part) {
  // Staged Q rows during the token loop, then the groups' sums (rows padded
  // by one float against bank conflicts): one buffer for both.
  constexpr int kQs = kSkTokens * R, kRed = kSkGroups * kSkCols * (R + 1);
  __shared__ float buf[kQs > kRed ? kQs : kRed];
  float(*qs)[R] = reinterpret_cast<float(*)[R]>(buf);
  float(*red)[kSkCols][R + 1] = reinterpret_cast<float(*)[kSkCols][R + 1]>(buf);
  const int c = threadIdx.x % kSkCols, g = threadIdx.x / kSkCols;
  const int i = blockIdx.x * kSkCols + c;
  const int t0 = blockIdx.y * kSkTokens;
  const int nt = min(kSkTokens, T - t0);
  // Stage Q rows [t0, t0 + nt) x [0, r), zero past r.
  for (int e = threadIdx.x; e < kSkTokens * R; e += blockDim.x) {
    const int tt = e / R, j = e % R;
    qs[tt][j] = (tt < nt && j < r) ? __bfloat162float(Q[(long long)(t0 + tt) * ldq + j]) : 0.f;
  }
  __syncthreads();
  float acc[R];
#pragma unroll
  for (int j = 0; j < R; ++j) acc[j] = 0.f;
  if (i < W) {
#pragma unroll 4
    for (int tt = g; tt < nt; tt += kSkGroups) {
      const float p = __bfloat162float(P[(long long)(t0 + tt) * ldp + i]);
#pragma unroll
      for (int j = 0; j < R; ++j) acc[j] = fmaf(p, qs[tt][j], acc[j]);
    }
  }
  __syncthreads();  // every thread is done with qs
#pragma unroll
  for (int j = 0; j < R; ++j) red[g][c][j] = acc[j];
  __syncthreads();
  // 64 columns x r outputs, summed over the four groups in order.
  for (int e = threadIdx.x; e < kSkCols * R; e += blockDim.x) {
    const int cc = e / R, j = e % R;
    const int ii = blockIdx.x * kSkCols + cc;
    if (ii < W && j < r) {
      const float s = red[0][cc][j] + red[1][cc][j] + red[2][cc][j] + red[3][cc][j];
      part[((long long)blockIdx.y * W + ii) * r + j] = s;
    }
  }
}

}  // namespace

int skinny_token_blocks(int64_t T) { return (int)std::max<int64_t>(1, (T + kSkTokens - 1) / kSkTokens); }

cudaError_t skinny_tn(const void* P, int ldp, const void* Q, int ldq, int T, int W, int r, float* part,
                      const char* name, cudaStream_t st) {
  const dim3 grid((unsigned)((W + kSkCols - 1) / kSkCols), (unsigned)skinny_token_blocks(T));
  const auto* p = reinterpret_cast<const __nv_bfloat16*>(P);
  const auto* q = reinterpret_cast<const __nv_bfloat16*>(Q);
  ProfRange pr(name, st);
  if (r <= 8)
    skinny_tn_kernel<8><<<grid, 256, 0, st>>>(p, ldp, q, ldq, T, W, r, part);
  else if (r <= 16)
    skinny_tn_kernel<16><<<grid, 256, 0, st>>>(p, ldp, q, ldq, T, W, r, part);
  else if (r <= 32)
    skinny_tn_kernel<32><<<grid, 256, 0, st>>>(p, ldp, q, ldq, T, W, r, part);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace dora
