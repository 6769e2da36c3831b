"""Host-side planning of the fused decode kernel, checked on the CPU.

The fused decode kernel (decode_fused.cu) computes its shared-memory plan,
activation fragment order and per-CTA jobs (computed from their number) with
host/device functions.
A small host program (compiled with nvcc, run without a GPU) evaluates them
over every shape the kernel accepts and checks the invariants the kernel
relies on: every fp16 activation has exactly one place in the fragment
order, and the four-at-a-time stores put each value there; the plan fits the
per-CTA shared-memory limit with 16-byte aligned regions; over all CTAs of
the grid, for every count of picked experts, every router row, every K part
of every gate/up tile and every output row of every expert (the shared one
included) is covered exactly once; job fields fit their widths; local tile
indices stay inside the reduction slots; and the workspace holds the
counters, logits and intermediate activations the kernel writes.
"""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_quantized_moe_gemv_b200", "csrc")

PROGRAM = r"""
#include "decode_fused.cu"
#include <cstdio>
#include <vector>
void moe::count_launches(int) {}
// the prefill scratch regions are not used by the decode kernel
size_t moe::grouped_ws_bytes(long long, int, int, int, int, bool) { return 0; }
size_t moe::router_tc_ws_bytes(long long, int, int) { return 0; }
using namespace moe;
using namespace moe::dfx;
template <int F>
int check_quads(int T, int K) {
  int bad = 0;
  for (int t = 0; t < T; ++t)
    for (int k0 = 0; k0 < K; k0 += 4)
      for (int i = 0; i < 4; ++i)
        if (frag_pos(F, k0 + i, t, T) != frag_pos(F, k0, t, T) + quad_off<F>(i)) ++bad;
  return bad;
}
int main() {
  int bad_frag = 0, bad_plan = 0, bad_cover = 0, bad_fields = 0, bad_ws = 0, eligible = 0, checked = 0;
  // fragment order: a bijection of (k, t) onto the fp16 places of the buffer,
  // and the four-at-a-time stores land where frag_pos puts each value
  for (int f = 1; f <= 3; ++f)
    for (int T = 1; T <= 4; ++T)
      for (int K = 256; K <= 2048; K += 256) {
        std::vector<int> seen(K * T, 0);
        for (int t = 0; t < T; ++t)
          for (int k = 0; k < K; ++k) {
            const int o = frag_pos(f, k, t, T);
            if (o < 0 || o % 2 || o / 2 >= K * T || seen[o / 2]++) ++bad_frag;
          }
      }
  for (int T = 1; T <= 4; ++T)
    for (int K = 256; K <= 2048; K += 256)
      bad_frag += check_quads<MOE_Q_INT4_SYM_G32>(T, K) + check_quads<MOE_Q_INT2_ASYM_G16>(T, K) +
                  check_quads<MOE_Q_INT8_PER_CHANNEL>(T, K);
  const int Gs[] = {148, 132};
  const int Es[] = {16, 24, 32, 64, 128, 256, 384, 512, 1024};
  const int Ks[] = {1, 2, 4, 6, 8, 10, 16};
  for (int G : Gs)
    for (int T = 1; T <= 4; ++T)
      for (int H = 256; H <= 2048; H += 256)
        for (int I = 256; I <= 2048; I += 256)
          for (int E : Es)
            for (int k : Ks) {
              if (k > E) continue;
              ++checked;
              if (!eligible_on(T, H, I, E, k, G)) continue;
              ++eligible;
              const Plan p = make_plan(T, H, I, E, k, G);
              const int offs[] = {p.o_x32, p.o_cand, p.o_hf, p.o_xf, p.o_rp, p.o_red, p.o_td, p.o_y, p.o_desc};
              for (int o : offs)
                if (o % 16) ++bad_plan;
              if (p.total + kStaticSmem > kSmemLimit) ++bad_plan;
              // staging buffers: aligned, and each warp's holds the largest
              // int4 / int2 job it may stage (a gate/up part or a down slice)
              if (p.o_stage >= 0) {
                if (p.o_stage % 16 || p.stage_bytes % 16 || p.o_stage + kWarps * p.stage_bytes > p.total) ++bad_plan;
                for (int f = MOE_Q_INT4_SYM_G32; f <= MOE_Q_INT2_ASYM_G16; ++f) {
                  const int nm = f == MOE_Q_INT2_ASYM_G16 ? 2 : 1;
                  const int ncols[2] = {H / kc(f) / gu_parts(H), I / kc(f)};
                  for (int ncol : ncols) {
                    int cp, sp;
                    stage_pitches(f, ncol, cp, sp);
                    if (16 * (cp + nm * sp) > p.stage_bytes || cp % 16 || sp % 16 ||
                        (ncol * (f == MOE_Q_INT2_ASYM_G16 ? 8 : 2)) % 16)
                      ++bad_plan;
                  }
                }
              }
              // every picked-expert count from 1 to the most, with and
              // without the shared expert and its gate row
              const int Umax = T * k < E ? T * k : E;
              const int ns = gu_parts(H);
              for (int U = 1; U <= Umax; U += (U < 4 ? 1 : 7)) {
                for (int v = 0; v < 2; ++v) {
                  const bool sh = v == 1, gate = v == 1;
                  const int ne = U + (sh ? 1 : 0);
                  std::vector<int> rows(E + 1, 0), parts(size_t(ne) * (I / 8) * ns, 0), outc(size_t(ne) * H, 0);
                  for (int b = 0; b < G; ++b) {
                    int e0, nrr;
                    router_range(E, G, b, e0, nrr);
                    const int na = phase_a_count(H, E, G, b, gate);
                    for (int j = 0; j < na; ++j) {
                      const Job jb = phase_a_job(H, j);
                      if (jb.kind != kRouter || jb.slot > nrr || (jb.slot == nrr && !(gate && b == G - 1)) ||
                          jb.part >= H / router_seg(H))
                        ++bad_fields;
                      else if (jb.part == 0)
                        rows[jb.slot == nrr ? E : e0 + jb.slot]++;
                    }
                    const int nb = phase_bc_count(H, I, G, b, U, sh);
                    int n0, nr;
                    out_rows(H, G, b, n0, nr);
                    if (nr > 16) ++bad_fields;
                    for (int j = 0; j < nb; ++j) {
                      const Job jb = phase_bc_job(H, I, G, b, U, sh, j);
                      const int e = jb.slot == kSharedSlot ? 0 : jb.slot + (sh ? 1 : 0);  // list position
                      if ((jb.slot == kSharedSlot && !sh) || (jb.slot != kSharedSlot && jb.slot >= U)) {
                        ++bad_fields;
                        continue;
                      }
                      if (jb.kind == kGateUp) {
                        if (jb.tile >= max_tiles(T, I, E, k, G) || jb.row0 % 8 || jb.row0 >= I || jb.part >= ns ||
                            jb.nrows != 16)
                          ++bad_fields;
                        else
                          parts[(size_t(e) * (I / 8) + jb.row0 / 8) * ns + jb.part]++;
                      } else if (jb.kind == kDown) {
                        if (jb.nrows != nr || jb.row0 != n0) ++bad_fields;
                        for (int r = 0; r < jb.nrows; ++r) outc[size_t(e) * H + jb.row0 + r]++;
                      } else {
                        ++bad_fields;
                      }
                    }
                  }
                  for (int e = 0; e < E; ++e)
                    if (rows[e] != 1) ++bad_cover;
                  if (rows[E] != (gate ? 1 : 0)) ++bad_cover;
                  for (size_t i = 0; i < parts.size(); ++i)
                    if (parts[i] != 1) ++bad_cover;
                  for (size_t i = 0; i < outc.size(); ++i)
                    if (outc[i] != 1) ++bad_cover;
                }
              }
              // the workspace the kernel writes: counters after the header,
              // logits [T, E] and h of every slot
              const WsLayout L = ws_layout(T, H, I, E, k);
              if (L.dcnt != 256 || size_t(kMaxSlots) * kCntStride * 4 > kDecodeCounterBytes ||
                  L.counts < L.dcnt + kDecodeCounterBytes || L.logits_u - L.logits < size_t(4) * T * E ||
                  L.shared_y - L.dh < decode_fused_ws_bytes(T, I) || L.dh % 256 || L.logits % 256)
                ++bad_ws;
            }
  printf("{\"bad_frag\": %d, \"bad_plan\": %d, \"bad_cover\": %d, \"bad_fields\": %d, \"bad_ws\": %d, "
         "\"eligible\": %d, \"checked\": %d, \"decode1\": %d, \"decode48\": %d, \"smem_decode1\": %d, "
         "\"smem_decode48\": %d, \"staged_decode1\": %d}\n",
         bad_frag, bad_plan, bad_cover, bad_fields, bad_ws, eligible, checked,
         int(eligible_on(1, 2048, 768, 512, 10, 148)), int(eligible_on(4, 2048, 768, 512, 10, 148)),
         make_plan(1, 2048, 768, 512, 10, 148).total, make_plan(4, 2048, 768, 512, 10, 148).total,
         int(make_plan(1, 2048, 768, 512, 10, 148).o_stage >= 0));
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
    r = subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(exe)], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_fragment_order_is_a_bijection(plan_report):
    assert plan_report["bad_frag"] == 0


def test_plans_fit_shared_memory_aligned(plan_report):
    assert plan_report["bad_plan"] == 0
    assert plan_report["eligible"] > 0


def test_jobs_cover_every_row_tile_and_output_once(plan_report):
    assert plan_report["bad_cover"] == 0


def test_job_fields_and_tile_slots_in_range(plan_report):
    assert plan_report["bad_fields"] == 0


def test_workspace_holds_what_the_kernel_writes(plan_report):
    assert plan_report["bad_ws"] == 0


def test_the_bench_decode_shapes_take_the_fused_kernel(plan_report):
    assert plan_report["decode1"] == 1 and plan_report["decode48"] == 1
    assert plan_report["staged_decode1"] == 1  # one-token decode stages its int4 rows
