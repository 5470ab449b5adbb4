// The side stream and event pool of the segmented launch sequences (host only).
#include <mutex>

#include "gdn_tc_common.cuh"

namespace gdn {
namespace tcx {

namespace {

constexpr int kMaxDevices = 64;
constexpr int kEvents = 4 * kMaxSeg + 8;

struct SideDev {
  std::mutex mu;
  bool tried = false, ok = false;
  cudaStream_t stream = nullptr;
  cudaEvent_t ev[kEvents] = {};
};

SideDev g_side[kMaxDevices];

}  // namespace

SideLock::SideLock() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  SideDev* d = &g_side[dev];
  d->mu.lock();
  dev_ = d;
  if (!d->tried) {
    d->tried = true;
    int least = 0, greatest = 0;
    bool good = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
                cudaStreamCreateWithPriority(&d->stream, cudaStreamNonBlocking, greatest) == cudaSuccess;
    for (int i = 0; good && i < kEvents; ++i)
      good = cudaEventCreateWithFlags(&d->ev[i], cudaEventDisableTiming) == cudaSuccess;
    d->ok = good;
  }
  ok_ = d->ok;
}

SideLock::~SideLock() {
  if (dev_) static_cast<SideDev*>(dev_)->mu.unlock();
}

cudaStream_t SideLock::stream() const { return static_cast<SideDev*>(dev_)->stream; }

cudaError_t SideLock::record(cudaStream_t st, cudaEvent_t* ev) {
  if (next_ >= kEvents) return cudaErrorInvalidValue;
  *ev = static_cast<SideDev*>(dev_)->ev[next_++];
  return cudaEventRecord(*ev, st);
}

cudaError_t SideLock::fork(cudaStream_t s) {
  cudaEvent_t ev;
  cudaError_t e = record(s, &ev);
  if (e != cudaSuccess) return e;
  return cudaStreamWaitEvent(stream(), ev, 0);
}

}  // namespace tcx
}  // namespace gdn
