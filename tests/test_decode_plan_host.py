"""Host-side planning of the fused decode kernel, checked on the CPU.

The decode kernel's shared-memory layout, slot geometry, K-piece split and
fragment order are computed by host/device functions in decode_stream.cu.
A small host program (compiled with nvcc, run without a GPU) evaluates them
over every shape the kernel accepts and checks the invariants the kernel
relies on: every fp16 activation has exactly one place in the fragment
order, tile pieces fit a slot, slot offsets are 16-byte aligned, the ring
has an even number of slots (one producer warp per slot), the whole plan
fits the per-CTA shared-memory limit, and the workspace regions it writes
(router partials, the activations of the picked experts) are large enough.
"""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_quantized_moe_gemv_b200", "csrc")

PROGRAM = r"""
#include "decode_stream.cu"
#include <cstdio>
#include <vector>
void moe::count_launches(int) {}
// the prefill scratch regions are not used by the decode kernel
size_t moe::grouped_ws_bytes(long long, int, int, int, int, bool) { return 0; }
size_t moe::router_tc_ws_bytes(long long, int, int) { return 0; }
using namespace moe;
using namespace moe::dks;
int main() {
  int bad_frag = 0, bad_geo = 0, bad_plan = 0, bad_ws = 0, eligible = 0, checked = 0;
  // fragment order: a bijection of (k, t) onto the fp16 slots of the buffer
  for (int fmt = 1; fmt <= 3; ++fmt)
    for (int T = 1; T <= 4; ++T)
      for (int K = 256; K <= 2048; K += 256) {
        std::vector<int> seen(frag_bytes(K, T) / 2, 0);
        for (int t = 0; t < T; ++t)
          for (int k = 0; k < K; ++k) {
            const int o = frag_off(fmt, k, t, T);
            if (o < 0 || o % 2 || o / 2 >= int(seen.size()) || seen[o / 2]++) ++bad_frag;
          }
      }
  // tile pieces: fit a slot, 16-byte aligned parts, odd 16-byte row strides
  for (int fmt = 1; fmt <= 3; ++fmt)
    for (int T = 1; T <= 4; ++T)
      for (int K = 256; K <= 2048; K += 256)
        for (int wb = 0; wb < 2; ++wb) {
          const int np = npieces(fmt, K, T, wb != 0);
          if (np == 0) { ++bad_geo; continue; }
          const Geo g = geo(fmt, K / np, T, wb != 0);
          if (g.bytes > kSlotBytes || g.cs % 16 || ((g.cs / 16) & 1) == 0 || g.aux0 % 16 || g.aux1 % 16 ||
              g.bofs % 16 || (g.as && (g.as % 16 || ((g.as / 16) & 1) == 0)))
            ++bad_geo;
        }
  // plans of every accepted shape
  const int Es[] = {16, 24, 32, 64, 128, 256, 384, 512, 1024};
  const int Ks[] = {1, 2, 4, 6, 8, 10, 16};
  for (int T = 1; T <= 4; ++T)
    for (int H = 256; H <= 2048; H += 256)
      for (int I = 256; I <= 2048; I += 256)
        for (int E : Es)
          for (int k : Ks) {
            if (k > E) continue;
            ++checked;
            if (!decode_stream_eligible(T, H, I, E, k)) continue;
            ++eligible;
            const int S = pick_slots(T, H, E, k);
            const Plan p = make_plan(T, H, E, k, S);
            if (S < 4 || S > kMaxSlots || S % kProducers || p.total + kStaticSmem > kSmemLimit ||
                p.o_slots % 1024 || kSlotBytes % 1024)
              ++bad_plan;
            // workspace regions the kernel writes: router partials [T, E, RQ] fp32 and the
            // fp16 activations of every picked expert plus the shared one
            const WsLayout L = ws_layout(T, H, I, E, k);
            if (L.h - L.partial < size_t(4) * T * E * router_rq(H) ||
                L.shared_y - L.h < decode_stream_hfrag_bytes(T, I, k) || L.partial % 256 || L.h % 256)
              ++bad_ws;
          }
  printf("{\"bad_frag\": %d, \"bad_geo\": %d, \"bad_plan\": %d, \"bad_ws\": %d, \"eligible\": %d, \"checked\": %d, "
         "\"slots_decode1\": %d, \"slots_decode48\": %d, \"decode1\": %d, \"decode48\": %d}\n",
         bad_frag, bad_geo, bad_plan, bad_ws, eligible, checked, pick_slots(1, 2048, 512, 10), pick_slots(4, 2048, 512, 10),
         int(decode_stream_eligible(1, 2048, 768, 512, 10)), int(decode_stream_eligible(4, 2048, 768, 512, 10)));
  return 0;
}
"""


@pytest.fixture(scope="module")
def plan_report(tmp_path_factory):
    if shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("decode_plan")
    src = d / "plan.cu"
    src.write_text(PROGRAM)
    exe = d / "plan"
    subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True, capture_output=True,
                   timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_fragment_order_is_a_bijection(plan_report):
    assert plan_report["bad_frag"] == 0


def test_tile_pieces_fit_and_are_aligned(plan_report):
    assert plan_report["bad_geo"] == 0


def test_plans_fit_shared_memory_with_an_even_ring(plan_report):
    assert plan_report["bad_plan"] == 0
    assert plan_report["eligible"] > 0


def test_workspace_holds_what_the_kernel_writes(plan_report):
    assert plan_report["bad_ws"] == 0


def test_the_bench_decode_shapes_take_the_fused_kernel(plan_report):
    assert plan_report["decode1"] == 1 and plan_report["decode48"] == 1
    assert plan_report["slots_decode1"] >= 4 and plan_report["slots_decode1"] % 2 == 0
    assert plan_report["slots_decode48"] >= 4 and plan_report["slots_decode48"] % 2 == 0
