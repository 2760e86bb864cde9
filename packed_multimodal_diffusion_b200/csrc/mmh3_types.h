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
};

struct DevStatus {
  int code;   // first DevErr recorded (0 = none)
  int site;   // kernel-specific detail (barrier index, iteration)
  int count;  // number of CTAs that recorded an error
  int pad;
};

// Segment table as a kernel parameter: token i reads modulation row
// row[k] where start[k] <= i < stop[k].
constexpr int kMaxSeg = 16;
struct SegRows {
  int n;
  int start[kMaxSeg];
  int stop[kMaxSeg];
  int row[kMaxSeg];
};

__host__ __device__ __forceinline__ int seg_row(const SegRows& s, int i) {
  int r = 0;
#pragma unroll
  for (int k = 0; k < kMaxSeg; ++k)
    if (k < s.n && i >= s.start[k] && i < s.stop[k]) r = s.row[k];
  return r;
}

}  // namespace mmh3
