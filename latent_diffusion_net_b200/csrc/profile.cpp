#include "profile.h"

#include <string.h>

#include <atomic>
#include <vector>

#include "sd_api.h"

namespace sdp {

namespace {

std::atomic<long long> g_launches{0};

struct Rec {
  char kernel[24];
  int family;
  int kernels;
  double flops, bytes;
};

struct Recorder {
  bool on = false;
  size_t idx = 0;
  long long kernels = 0;
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> ev;  // 2 per record, reused across recordings
};

thread_local Recorder t_rec;

bool capturing(cudaStream_t st) {
  cudaStreamCaptureStatus s = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &s) != cudaSuccess) return false;
  return s != cudaStreamCaptureStatusNone;
}

}  // namespace

Scope::Scope(const char* kernel, int family, double flops, double bytes, cudaStream_t st, int kernels)
    : slot_(-1), flags_(0), st_(st) {
  g_launches.fetch_add(kernels, std::memory_order_relaxed);
  Recorder& r = t_rec;
  if (!r.on) return;
  r.kernels += kernels;
  const size_t i = r.idx;
  if (2 * i + 1 >= r.ev.size()) {
    if (capturing(st)) return;  // events are only created outside capture
    while (r.ev.size() < 2 * i + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      r.ev.push_back(e);
    }
  }
  if (r.recs.size() <= i) r.recs.resize(i + 1);
  Rec& rc = r.recs[i];
  memset(rc.kernel, 0, sizeof(rc.kernel));
  strncpy(rc.kernel, kernel, sizeof(rc.kernel) - 1);
  rc.family = family;
  rc.kernels = kernels;
  rc.flops = flops;
  rc.bytes = bytes;
  // inside stream capture a plain event record only expresses a dependency;
  // the external flag turns it into an event-record node of the graph
  flags_ = capturing(st) ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (cudaEventRecordWithFlags(r.ev[2 * i], st, flags_) != cudaSuccess) return;
  slot_ = (int)i;
  r.idx = i + 1;
}

Scope::~Scope() {
  if (slot_ < 0) return;
  cudaEventRecordWithFlags(t_rec.ev[2 * slot_ + 1], st_, flags_);
}

}  // namespace sdp

extern "C" {

sd_status sd_profile_begin(void) {
  sdp::t_rec.on = true;
  sdp::t_rec.idx = 0;
  sdp::t_rec.kernels = 0;
  return SD_OK;
}

sd_status sd_profile_end(int32_t* n_kernels) {
  sdp::t_rec.on = false;
  if (n_kernels) *n_kernels = (int32_t)sdp::t_rec.kernels;
  return SD_OK;
}

sd_status sd_profile_read(sd_launch_record* out, int32_t capacity, int32_t* n) {
  sdp::Recorder& r = sdp::t_rec;
  if (n) *n = (int32_t)r.idx;
  if (!out) return SD_OK;
  if (capacity < (int32_t)r.idx) return SD_ERR_CAPACITY;
  for (size_t i = 0; i < r.idx; ++i) {
    sd_launch_record& o = out[i];
    memset(&o, 0, sizeof(o));
    memcpy(o.kernel, r.recs[i].kernel, sizeof(o.kernel));
    o.family = r.recs[i].family;
    o.kernels = r.recs[i].kernels;
    o.flops = r.recs[i].flops;
    o.bytes = r.recs[i].bytes;
    float ms = -1.f;
    if (cudaEventElapsedTime(&ms, r.ev[2 * i], r.ev[2 * i + 1]) != cudaSuccess) {
      (void)cudaGetLastError();
      ms = -1.f;
    }
    o.ms = ms;
  }
  return SD_OK;
}

int64_t sd_launch_count(void) { return sdp::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
