// Host-only probe of the library's launch planner (make_plan in csrc/dora_api.cu),
// for the CPU tests: compiled together with dora_api.cu by g++, with the device
// side replaced by stubs, it prints the plan of one call as a JSON line.
//
//   planner_probe d_out d_in r T op
//
// No GPU is involved: device_sm_count() falls back to the 148 SMs of a B200 when
// no device is visible, and the stub below answers the cluster-occupancy query
// with B200 figures (clusters of 2, 4, 6, 8 and 16 CTAs resident at once; those of
// 4, 6 and 8 CTAs are the runtime's answers on this machine's B200s, the others the
// pair count and a conservative guess). The kernels' entry points are never
// called; their stubs only satisfy the linker.
#include <cstdio>
#include <cstdlib>

#include "dora_internal.h"

namespace dora {

int max_active_pair_clusters(int cs) {
  switch (cs) {
    case 1: return 74;
    case 2: return 33;
    case 3: return 22;
    case 4: return 15;
    case 8: return 7;
    default: return 0;
  }
}

// Entry points of the other translation units: never called by the probe.
dora_status_t bf16_norm(const dora_desc_t&, const Plan&, const void*, const void*, const void*, const float*, float*,
                        float*, float*, uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t bf16_forward(const dora_desc_t&, const Plan&, int64_t, const void*, const void*, const void*,
                           const void*, const float*, void*, void*, void*, uint8_t*, cudaStream_t) {
  return DORA_EUNSUPPORTED;
}
dora_status_t bf16_backward(const dora_desc_t&, const Plan&, int64_t, const void*, const void*, const void*,
                            const void*, const void*, const float*, const float*, const void*, const void*, float*,
                            void*, void*, void*, uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t bf16_backward_full(const dora_desc_t&, const Plan&, int64_t, const void*, const void*, const void*,
                                 const void*, const void*, const float*, const float*, const void*, const void*,
                                 float*, void*, void*, void*, uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t bf16_merge(const dora_desc_t&, const Plan&, const void*, const void*, const void*, const float*, void*,
                         uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t f32_norm(const dora_desc_t&, const Plan&, const float*, const float*, const float*, const float*,
                       float*, float*, float*, uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t f32_forward(const dora_desc_t&, const Plan&, int64_t, const float*, const float*, const float*,
                          const float*, const float*, float*, float*, float*, uint8_t*, cudaStream_t) {
  return DORA_EUNSUPPORTED;
}
dora_status_t f32_backward(const dora_desc_t&, const Plan&, int64_t, const float*, const float*, const float*,
                           const float*, const float*, const float*, const float*, const float*, const float*,
                           float*, float*, float*, float*, uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t f32_backward_full(const dora_desc_t&, const Plan&, int64_t, const float*, const float*, const float*,
                                const float*, const float*, const float*, const float*, const float*, const float*,
                                float*, float*, float*, float*, uint8_t*, cudaStream_t) {
  return DORA_EUNSUPPORTED;
}
dora_status_t f32_merge(const dora_desc_t&, const float*, const float*, const float*, const float*, float*,
                        cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t vera_compose(const dora_desc_t&, const void*, const float*, const float*, void*, cudaStream_t) {
  return DORA_EUNSUPPORTED;
}
dora_status_t vera_grad(const dora_desc_t&, const Plan&, const void*, const float*, const float*, const void*, float*,
                        float*, uint8_t*, cudaStream_t) { return DORA_EUNSUPPORTED; }
dora_status_t selftest_timeout(uint32_t, unsigned int*, cudaStream_t) { return DORA_EUNSUPPORTED; }
cudaError_t read_and_clear_device_status(cudaStream_t, unsigned int*) { return cudaErrorNotSupported; }

}  // namespace dora

int main(int argc, char** argv) {
  if (argc != 6) {
    std::fprintf(stderr, "usage: %s d_out d_in r T op\n", argv[0]);
    return 2;
  }
  dora_desc_t d{};
  d.d_out = std::atoll(argv[1]);
  d.d_in = std::atoll(argv[2]);
  d.r = std::atoll(argv[3]);
  d.dtype = DORA_BF16;
  d.s = 0.5f;
  const int64_t T = std::atoll(argv[4]);
  const int op = std::atoi(argv[5]);
  const dora::Plan p = dora::make_plan(d, T, op);
  std::printf(
      "{\"sms\": %d, \"norm_splits\": %d, \"norm_kb_per_split\": %d, \"norm_bn\": %d, \"u_bn\": %d, \"u_cs\": %d, "
      "\"fwd_cs\": %d, \"fwd_defer\": %d, \"fwd_pairs\": %d, \"du_bn\": %d, \"du_cs\": %d, \"dB_bn\": %d, "
      "\"dx_cs\": %d, \"dBA_grouped\": %d, \"bwd_fork\": %d, \"dx_pairs\": %d, \"dBA_pairs\": %d, \"dx_defer\": %d, "
      "\"total\": %zu}\n",
      p.sms, p.norm.splits, p.norm.kb_per_split, p.norm_bn, p.u_bn, p.u_cs, p.fwd_cs, p.fwd_defer, p.fwd_pairs,
      p.du_bn, p.du_cs, p.dB_bn, p.dx_cs, p.dBA_grouped, p.bwd_fork, p.dx_pairs, p.dBA_pairs, p.dx_defer, p.total);
  return 0;
}
