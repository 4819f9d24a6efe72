// pipe_schedule.h -- host-only: the chunk schedule of the host-buffer calls
// (sage_attn_fwd_host, sage_attn_fwd_nvfp4_host).  No CUDA; compiled into
// the library and, on its own, by the CPU tests that check the schedule.
#pragma once

#include <algorithm>
#include <cstdint>

namespace sage {

// KV-head groups of the chunk that starts at group g0 of batch entry b.
//
// The call has B batch entries of Hkv groups each. Chunks hold up to gpc
// groups and never span two batch entries.
//
// With `edge`, the first chunk of the call and its last chunk hold a single
// group each:
// - copying the first chunk in is the only copy that no kernel overlaps;
// - the last chunk's kernels and its copy back run after every copy in has
//   ended.
// Small edge chunks make both short. The chunks between them keep gpc groups,
// and the last batch entry leaves its final group to a chunk of its own.
inline int64_t pipe_chunk_groups(int64_t b, int64_t g0, int64_t B, int64_t Hkv, int64_t gpc,
                                 bool edge) {
  const int64_t left = Hkv - g0;
  int64_t ng = std::min(gpc, left);
  if (edge) {
    if (b == 0 && g0 == 0) return 1;
    if (b == B - 1 && left > 1 && left <= gpc) ng = left - 1;
  }
  return ng;
}

}  // namespace sage
