// Plain data types shared by host and device code of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mmh3 {

// ---------------------------------------------------------------- status word
// Device-side error codes written by a kernel that gave up waiting.  The host
// reads them after a stream synchronisation (mmh3_device_status).
enum DevErr : int {
  DEV_OK = 0,
  DEV_TIMEOUT_PRODUCER = 1,
  DEV_TIMEOUT_MMA = 2,
  DEV_TIMEOUT_EPILOGUE = 3,
  DEV_TIMEOUT_SOFTMAX = 4,
  DEV_TIMEOUT_SELFTEST = 5,
  // checks of the MMH3_CHECK mode (recorded, never trapped)
  DEV_CHECK_ROW = 6,     // a token's modulation row outside [0, rows)
  DEV_CHECK_TMA = 7,     // a TMA copy at an unaligned or negative coordinate
  DEV_CHECK_CANARY = 8,  // a workspace canary overwritten (site: kernel * 16 + region)
  DEV_TIMEOUT_COPY = 9,  // a bulk row copy that never landed (site: the row)
};

__host__ __device__ __forceinline__ bool dev_err_is_check(int code) {
  return code >= DEV_CHECK_ROW && code <= DEV_CHECK_CANARY;
}

struct DevStatus {
  int code;   // first DevErr recorded (0 = none)
  int site;   // kernel-specific detail (barrier index, iteration)
  int count;  // number of CTAs that recorded an error
  int check;  // 1: the MMH3_CHECK mode's device checks are on (host-written)
};

// Segment table as a kernel parameter: token i reads modulation row
// row[k] where start[k] <= i < stop[k].  limit > 0 (MMH3_CHECK mode): a row
// outside [0, limit) is recorded in *status and replaced by row 0.
constexpr int kMaxSeg = 16;
struct SegRows {
  int n;
  int start[kMaxSeg];
  int stop[kMaxSeg];
  int row[kMaxSeg];
  int limit;
  DevStatus* status;
};

__host__ __device__ __forceinline__ int seg_row(const SegRows& s, int i) {
  int r = 0;
#pragma unroll
  for (int k = 0; k < kMaxSeg; ++k)
    if (k < s.n && i >= s.start[k] && i < s.stop[k]) r = s.row[k];
  return r;
}

#ifdef __CUDACC__
__device__ __forceinline__ int seg_row_checked(const SegRows& s, int i) {
  int r = seg_row(s, i);
  if (s.limit > 0 && (r < 0 || r >= s.limit)) {
    if (s.status != nullptr && atomicCAS(&s.status->code, 0, (int)DEV_CHECK_ROW) == 0) s.status->site = i;
    if (s.status != nullptr) atomicAdd(&s.status->count, 1);
    r = 0;
  }
  return r;
}
#endif

}  // namespace mmh3
