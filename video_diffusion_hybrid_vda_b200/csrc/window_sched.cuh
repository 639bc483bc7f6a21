// Host plan of the window-and-anchor Softmax ("Video DeltaNet", 10100.com
// article, 方法概述 item 1), shared by its kernels: consecutive query frames
// with the same visible key set form a segment, whose keys are at most three
// contiguous token intervals (the window, frame 0, frame T-1).  The plan is
// built on the host and passed to a kernel by value.
#pragma once

#include <stdint.h>

#include "../../include/vdn.h"

namespace vdn {

constexpr int kMaxSegs = 256;

struct WinSeg {
  int q0, q1;      // query token rows [q0, q1)
  int tile_base;   // first CTA tile index of this segment (launch order)
  int ntiles;      // 256-row CTA tiles
  int pair_base;   // first CTA-pair index of this segment (pair kernel)
  int npairs;      // 512-row CTA pairs
  int nint;        // key intervals (1..3)
  int k0[3], k1[3];
  int nkv;         // 128-key tiles over all intervals
};

struct WinSched {
  int nseg;
  int total_tiles;
  int total_pairs;
  WinSeg seg[kMaxSegs];
};

// Segments ordered heaviest first; false when the mask needs more segments
// or intervals than the tables hold.
bool build_schedule(const vdn_shape& s, int cf, int wc, unsigned anchors, WinSched* out);

// The key intervals of one segment, held in registers, and a cursor over
// its key tiles of STEP keys (start row, number of valid keys).
struct KvRange {
  int nint, a0, a1, a2, b0, b1, b2;
  int mctx;  // context (text/audio) keys, visible to every query, after the video keys
  __device__ void load(const WinSeg& s, int m_ctx) {
    mctx = m_ctx;
    nint = s.nint;
    a0 = s.k0[0];
    a1 = s.k0[1];
    a2 = s.k0[2];
    b0 = s.k1[0];
    b1 = s.k1[1];
    b2 = s.k1[2];
  }
  __device__ int start(int iv) const { return iv == 0 ? a0 : (iv == 1 ? a1 : a2); }
  __device__ int end(int iv) const { return iv == 0 ? b0 : (iv == 1 ? b1 : b2); }
};

template <int STEP>
struct KvCursorT {
  int iv, pos, end;
  bool ctx;  // true once the cursor walks the context keys
  __device__ void init(const KvRange& r) {
    iv = 0;
    pos = r.a0;
    end = r.b0;
    ctx = false;
  }
  __device__ void next(const KvRange& r) {
    pos += STEP;
    if (pos >= end && !ctx) {
      if (iv + 1 < r.nint) {
        ++iv;
        pos = r.start(iv);
        end = r.end(iv);
      } else if (r.mctx > 0) {
        ctx = true;
        pos = 0;
        end = r.mctx;
      }
    }
  }
  __device__ int valid() const { return min(STEP, end - pos); }
};
using KvCursor = KvCursorT<128>;

}  // namespace vdn
