"""The chunk schedule of the host-buffer calls (csrc/pipe_schedule.h, the
header the library itself includes), compiled on its own with g++ and walked
the way run_host_pipeline walks it.

For every shape tried, the chunks must tile every (batch entry, KV-head
group) exactly once, in order. Each chunk holds between 1 and gpc groups and
stays inside one batch entry. With the edge rule, the call's first and last
chunks hold one group each. This is what makes the chunked result the
one-shot result: every group is a problem of its own, and each is computed
exactly once."""
import os
import subprocess

import quantized_attention_05_b200 as S

HEADER_DIR = os.path.join(os.path.dirname(S.__file__), "csrc")

SRC = r"""
#include <cstdio>
#include <vector>
#include "pipe_schedule.h"
using sage::pipe_chunk_groups;
int main() {
  long bad = 0, calls = 0;
  for (int64_t B = 1; B <= 5; ++B)
    for (int64_t Hkv = 1; Hkv <= 17; ++Hkv)
      for (int64_t gpc = 1; gpc <= Hkv; ++gpc)
        for (int e = 0; e < 2; ++e) {
          const bool edge = e != 0;
          std::vector<int> seen(B * Hkv, 0);
          std::vector<int64_t> sizes;
          for (int64_t b = 0; b < B; ++b)
            for (int64_t g0 = 0, ng = 0; g0 < Hkv; g0 += ng) {
              ng = pipe_chunk_groups(b, g0, B, Hkv, gpc, edge);
              if (ng < 1 || ng > gpc || g0 + ng > Hkv) { ++bad; ng = 1; }
              for (int64_t g = g0; g < g0 + ng && g < Hkv; ++g) seen[b * Hkv + g]++;
              sizes.push_back(ng);
            }
          for (int s : seen) bad += s != 1;
          if (edge && B * Hkv > 1) bad += sizes.front() != 1 || sizes.back() != 1;
          if (!edge) {                       // uniform chunks, a ragged end per batch entry
            int64_t k = 0;
            for (int64_t b = 0; b < B; ++b)
              for (int64_t g0 = 0; g0 < Hkv; g0 += gpc) bad += sizes[k++] != std::min(gpc, Hkv - g0);
          }
          ++calls;
        }
  std::printf("%ld %ld\n", calls, bad);
  return bad != 0;
}
"""


def test_chunk_schedule_tiles_every_group_once(tmp_path):
    src = tmp_path / "sched.cpp"
    src.write_text(SRC)
    exe = tmp_path / "sched"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", HEADER_DIR, str(src), "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    calls, bad = map(int, r.stdout.split())
    assert calls > 1000 and bad == 0 and r.returncode == 0


def test_host_workspace_covers_the_edge_chunks():
    """The automatic schedule of the causal GQA workload (B=4, Hkv=8, four
    groups per chunk) uses chunks of 1, 4, 3, ..., 3, 1 groups; the workspace
    is the three slots plus the largest of their per-chunk workspaces (the
    four-group one here)."""
    L = S.lib()
    B_, Hq, Hkv, N, D = 4, 32, 8, 16384, 128
    auto = L.sage_attn_fwd_host_workspace_bytes(B_, Hq, Hkv, N, N, D, None, 0)
    four = L.sage_attn_fwd_host_workspace_bytes(B_, Hq, Hkv, N, N, D, None, 4)
    assert auto == four
