// Internal declarations shared by the C ABI (dora_api.cu) and the bf16 / fp32
// implementations. Nothing here is exported.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>

#include <cuda_runtime.h>

#include "../../include/dora.h"

namespace dora {

// Workspace plan: every offset a call will use, computed from (desc, T, op)
// and the device's SM count alone, so dora_workspace_size() and the call agree.
struct Split {
  int splits = 1;
  int kb_per_split = 0;
};

struct Plan {
  int sms = 148;
  // norm
  Split norm;
  int norm_bn = 0;
  size_t off_gs = 0, off_norm_part = 0;
  // forward: u = s x A^T on CTA-pair clusters (tile width, pairs per cluster = K splits);
  // the base GEMM persistent (fwd_cs = 0) or, for few tiles, on clusters of fwd_cs pairs
  int u_bn = 0, u_cs = 1, fwd_cs = 0;
  // the base GEMM launched beside u (both fit on the SMs at once): it waits for u only
  // before its su k-block
  int fwd_defer = 0;
  // pairs the persistent base GEMM runs on (fewer than the device's when u runs beside it)
  int fwd_pairs = 74;
  size_t off_su = 0;
  // backward: du, dB, dA on pair clusters; dx like the base GEMM
  int dm_rowblocks = 0, dm_rows = 256;
  // (dB_grouped: dB and dA in one grouped launch of whole tiles, both dB_bn wide)
  int du_bn = 0, du_cs = 1, dB_bn = 0, dB_cs = 1, dA_bn = 0, dA_cs = 1, dx_cs = 0, dBA_grouped = 0;
  // dx and the grouped dB/dA launch both follow du alone; when dx's tiles leave SM pairs
  // free (bwd_fork), the two run at once on two streams, dx on dx_pairs pairs and dB/dA on
  // dBA_pairs (dx on the second stream, or, with dx_defer, dB/dA there)
  int bwd_fork = 0, dx_pairs = 0, dBA_pairs = 0;
  // under the fork, dx also starts beside du when both fit on the SMs at once (dx_defer);
  // dB/dA then take a second copy of du (off_du2), computed on their own stream
  int dx_defer = 0;
  size_t off_dz = 0, off_dm_part = 0, off_du = 0, off_du2 = 0;
  // full (non-detached) gradient: kappa, kappa-scaled B, Gram, Q = W' A^T, H = s B^T diag(kappa) B
  Split q, h;
  int q_bn = 0, h_bn = 0;
  size_t off_kappa = 0, off_bk = 0, off_q_part = 0, off_h_part = 0, off_h = 0;
  // DVoRA gradient: row blocks of the dd partial sums (scratch in off_f32_a)
  int vera_blocks = 0;
  // split counters (+ padding that must start at zero), cleared once per call
  size_t off_ctr = 0, zero_bytes = 0;
  // fp32 path scratch
  size_t off_f32_a = 0, off_f32_b = 0, off_f32_c = 0;
  size_t total = 0;
};

// Whole-rank tile width for CTA-pair GEMMs with K-major B (widths 64 .. 512).
inline int bn_pair_k(int64_t r) { return r <= 64 ? 64 : r <= 128 ? 128 : r <= 256 ? 256 : r <= 384 ? 384 : 512; }

int device_sm_count();
// Clusters of cs CTA pairs (cs = 1..4, one CTA per SM) the current device holds at once; 0 if unknown.
int max_active_pair_clusters(int cs);
Plan make_plan(const dora_desc_t& d, int64_t T, int op);

// Thread-local error message for dora_last_error().
void set_error(const std::string& msg);

// Status word written by kernels whose bounded waits ran out.
cudaError_t read_and_clear_device_status(cudaStream_t st, unsigned int* out);
// One kernel whose bounded wait runs out after limit_us (failure-detection test).
dora_status_t selftest_timeout(uint32_t limit_us, unsigned int* scratch, cudaStream_t st);

// bf16 path (tcgen05 / TMA kernels)
dora_status_t bf16_norm(const dora_desc_t& d, const Plan& p, const void* W0, const void* A, const void* B,
                        const float* m, float* C, float* g, float* gm1, uint8_t* ws, cudaStream_t st);
dora_status_t bf16_forward(const dora_desc_t& d, const Plan& p, int64_t T, const void* x, const void* W0,
                           const void* A, const void* B, const float* gm1, void* y, void* su_save,
                           void* pre_save, uint8_t* ws, cudaStream_t st);
dora_status_t bf16_backward(const dora_desc_t& d, const Plan& p, int64_t T, const void* dy, const void* x,
                            const void* W0, const void* A, const void* B, const float* C, const float* g,
                            const void* su, const void* pre, float* dm, void* dA, void* dB, void* dx,
                            uint8_t* ws, cudaStream_t st);

dora_status_t bf16_backward_full(const dora_desc_t& d, const Plan& p, int64_t T, const void* dy, const void* x,
                                 const void* W0, const void* A, const void* B, const float* C, const float* g,
                                 const void* su, const void* pre, float* dm, void* dA, void* dB, void* dx,
                                 uint8_t* ws, cudaStream_t st);

dora_status_t bf16_merge(const dora_desc_t& d, const Plan& p, const void* W0, const void* A, const void* B,
                         const float* g, void* W_out, uint8_t* ws, cudaStream_t st);

// fp32 path (SIMT kernels)
dora_status_t f32_norm(const dora_desc_t& d, const Plan& p, const float* W0, const float* A, const float* B,
                       const float* m, float* C, float* g, float* gm1, uint8_t* ws, cudaStream_t st);
dora_status_t f32_forward(const dora_desc_t& d, const Plan& p, int64_t T, const float* x, const float* W0,
                          const float* A, const float* B, const float* gm1, float* y, float* su_save,
                          float* pre_save, uint8_t* ws, cudaStream_t st);
dora_status_t f32_backward(const dora_desc_t& d, const Plan& p, int64_t T, const float* dy, const float* x,
                           const float* W0, const float* A, const float* B, const float* C, const float* g,
                           const float* su, const float* pre, float* dm, float* dA, float* dB, float* dx,
                           uint8_t* ws, cudaStream_t st);

dora_status_t f32_backward_full(const dora_desc_t& d, const Plan& p, int64_t T, const float* dy, const float* x,
                                const float* W0, const float* A, const float* B, const float* C, const float* g,
                                const float* su, const float* pre, float* dm, float* dA, float* dB, float* dx,
                                uint8_t* ws, cudaStream_t st);

// DVoRA (both dtypes): B' = diag(b) B_shared diag(d), and db, dd from dB'.
dora_status_t vera_compose(const dora_desc_t& d, const void* Bs, const float* b, const float* dv, void* Bp,
                           cudaStream_t st);
dora_status_t vera_grad(const dora_desc_t& d, const Plan& p, const void* Bs, const float* b, const float* dv,
                        const void* dBp, float* db, float* dd, uint8_t* ws, cudaStream_t st);

// True while the kernel profiler is on (dora_profile_start .. dora_profile_stop):
// launches then drop programmatic dependent launch, so that the events around
// each kernel time that kernel alone.
bool profiling_on();

// Brackets one kernel launch with profiling events when profiling is on.
class ProfRange {
 public:
  ProfRange(const char* name, cudaStream_t st);
  ~ProfRange();
  ProfRange(const ProfRange&) = delete;
  ProfRange& operator=(const ProfRange&) = delete;

 private:
  cudaStream_t st_;
  int idx_;
};

dora_status_t f32_merge(const dora_desc_t& d, const float* W0, const float* A, const float* B, const float* g,
                        float* W_out, cudaStream_t st);

inline dora_status_t cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return DORA_OK;
  set_error(std::string(where) + ": " + cudaGetErrorString(e));
  return DORA_ECUDA;
}

}  // namespace dora
