// Per-device internal streams and events (created once per device, on first use).
#include "common.cuh"

namespace gptq2d {

namespace {
DevStreams g_dev[kMaxDevices];
}  // namespace

int dev_streams(DevStreams** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPTQ2D_ERR_CUDA;
  DevStreams& d = g_dev[dev];
  std::lock_guard<std::recursive_mutex> lk(d.mu);
  if (!d.ready) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return GPTQ2D_ERR_CUDA;
    if (cudaStreamCreateWithPriority(&d.hi, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&d.lo, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaStreamCreateWithPriority(&d.hi2, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&d.lo2, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaStreamCreateWithPriority(&d.hi3, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&d.lo3, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaStreamCreateWithFlags(&d.blk_p, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&d.blk_q, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&d.cp, cudaStreamNonBlocking) != cudaSuccess)
      return GPTQ2D_ERR_CUDA;
    cudaEvent_t* evs[] = {&d.fork,         &d.setup,        &d.join_hi,      &d.join_lo,
                          &d.join_hi2,     &d.join_lo2,     &d.join_hi3,     &d.join_lo3,
                          &d.cp_ev[0],     &d.cp_ev[1],     &d.cp_ev[2],     &d.q_ev[0],
                          &d.q_ev[1],      &d.q_ev[2],      &d.q_ev[3],      &d.blk_start,
                          &d.blk_prep[0],  &d.blk_prep[1],  &d.blk_quant[0], &d.blk_quant[1],
                          &d.blk_end[0],   &d.blk_end[1]};
    for (auto* e : evs)
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return GPTQ2D_ERR_CUDA;
    for (int r = 0; r < RING; ++r)
      if (cudaEventCreateWithFlags(&d.sw[r], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.far[r], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.farb[r], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.panel_done[0][r], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.panel_done[1][r], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.rest_done[0][r], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.rest_done[1][r], cudaEventDisableTiming) != cudaSuccess)
        return GPTQ2D_ERR_CUDA;
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    d.ready = true;
  }
  *out = &d;
  return GPTQ2D_OK;
}

}  // namespace gptq2d
