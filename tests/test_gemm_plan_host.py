"""Host-side sizing of the prefill grouped GEMM, checked on the CPU.

A host program (nvcc, no GPU) includes expert_gemm_sm100.cu and checks what
the kernels rely on: the dynamic shared memory of both dequantising GEMMs
(stage ring plus the dequant warps' raw-code staging) and of the wide-tile
GEMMs (stage ring plus the epilogue warps' scratch) fits the per-CTA limit, the row-tile bound
covers every routing, the heavy-slot bound covers every routing's groups
of more than one row tile (up to the slot cap), and the split of the row
tiles between the three GEMMs (wide tiles of the heavy groups, the
mma.sync GEMV for int4 groups of at most kMmaRows rows, the dequantising
GEMM for the rest, per group_lists) covers every row tile exactly once, on
seeded random routings with a skewed expert popularity.
"""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_quantized_moe_gemv_b200", "csrc")

PROGRAM = r"""
#include "expert_gemm_sm100.cu"
#include <cstdio>
#include <random>
#include <vector>
void moe::count_launches(int) {}
using namespace moe;
using namespace moe::gemm;
int main() {
  const size_t limit = 227 * 1024;
  const size_t smem_gu = size_t(Cfg<true>::kStages) * Cfg<true>::kStageBytes + size_t(kRawDepth) * kRawSlotBytes + 1024;
  const size_t smem_dn = size_t(Cfg<false>::kStages) * Cfg<false>::kStageBytes + size_t(kRawDepth) * kRawSlotBytes + 1024;
  const size_t smem_w = wide_smem_bytes<kGuNA, kGuNB>() > wide_smem_bytes<kDnNA, kDnNB>() ? wide_smem_bytes<kGuNA, kGuNB>() : wide_smem_bytes<kDnNA, kDnNB>();
  int bad_tiles = 0, bad_heavy = 0, bad_split = 0, cases = 0, n_wide = 0, n_mma = 0, n_light = 0;
  std::mt19937 rng(12345);
  const int Ts[] = {5, 37, 300, 1000, 8192};
  const int Es[] = {8, 64, 512};
  const int ks[] = {1, 2, 10};
  for (int T : Ts)
    for (int E : Es)
      for (int k : ks) {
        if (k > E) continue;
        for (int rep = 0; rep < 4; ++rep) {
          // k distinct experts per token, drawn with a Zipf-like skew (rep 0: uniform)
          std::vector<long long> cnt(E, 0);
          std::vector<double> wgt(E);
          for (int e = 0; e < E; ++e) wgt[e] = rep == 0 ? 1.0 : 1.0 / std::pow(double(e + 1), 0.5 * rep);
          for (int t = 0; t < T; ++t) {
            std::vector<double> w = wgt;
            for (int j = 0; j < k; ++j) {
              std::discrete_distribution<int> d(w.begin(), w.end());
              const int e = d(rng);
              ++cnt[e];
              w[e] = 0.0;
            }
          }
          for (int sh = 0; sh < 2; ++sh) {
            ++cases;
            long long tiles = 0, heavy = 0;
            for (int e = 0; e < E; ++e) {
              tiles += (cnt[e] + BN - 1) / BN;
              heavy += cnt[e] >= kHeavyRows;
            }
            if (sh) {
              tiles += (T + BN - 1) / BN;
              heavy += T >= kHeavyRows;
            }
            if (tiles > grouped_max_tiles(T, k, E, sh != 0)) ++bad_tiles;
            const long long cap = heavy < kMaxHeavy ? heavy : kMaxHeavy;
            if (cap > grouped_heavy_slots(T, k, sh != 0, 2048, 768)) ++bad_heavy;
            // the plan's split of the row tiles: slots in group order up to
            // the cap, every group's tiles in exactly one list
            const int max_heavy = grouped_heavy_slots(T, k, sh != 0, 2048, 768);
            int slots = 0;
            for (int gi = 0; gi < E + sh; ++gi) {
              const int n = gi < E ? int(cnt[gi]) : T;
              const int nt = (n + BN - 1) / BN;
              const bool slot = nt >= 2 && slots < max_heavy;
              if (nt >= 2) ++slots;
              const bool int4 = ((gi * 7 + rep) % 10) < 7;  // a mix of formats
              const GroupLists gl = group_lists(n, slot, int4);
              std::vector<int> cover(nt, 0);
              for (int j = 0; j < gl.nw; ++j) {
                ++cover[2 * j];
                if (2 * j + 1 < nt) ++cover[2 * j + 1];
              }
              for (int t = 0; t < gl.nl; ++t) ++cover[t];
              for (int t = 0; t < gl.nm; ++t) ++cover[t];
              for (int t = 0; t < nt; ++t) bad_split += cover[t] != 1;
              if (gl.nw && !slot) ++bad_split;
              if (gl.nm && (nt != 1 || n > kMmaRows || !int4 || slot)) ++bad_split;
              n_wide += gl.nw;
              n_mma += gl.nm;
              n_light += gl.nl;
            }
          }
        }
      }
  printf("{\"smem_gu\": %zu, \"smem_dn\": %zu, \"smem_w\": %zu, \"limit\": %zu, \"bad_tiles\": %d, \"bad_heavy\": %d, "
         "\"bad_split\": %d, \"n_wide\": %d, \"n_mma\": %d, \"n_light\": %d, \"cases\": %d, "
         "\"ws_8k\": %zu, \"ws_32k\": %zu}\n",
         smem_gu, smem_dn, smem_w, limit, bad_tiles, bad_heavy, bad_split, n_wide, n_mma, n_light, cases,
         grouped_ws_bytes(8192, 2048, 768, 10, 512, true),
         grouped_ws_bytes(32768, 2048, 768, 10, 512, true));
  return 0;
}
"""


@pytest.fixture(scope="module")
def report(tmp_path_factory):
    if shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("gemm_plan")
    src = d / "plan.cu"
    src.write_text(PROGRAM)
    exe = d / "plan"
    subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True, capture_output=True,
                   timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_every_gemm_fits_shared_memory(report):
    assert report["smem_gu"] <= report["limit"] and report["smem_dn"] <= report["limit"]
    assert report["smem_w"] <= report["limit"]


def test_row_tile_bound_covers_every_routing(report):
    assert report["cases"] > 0 and report["bad_tiles"] == 0


def test_heavy_slot_bound_covers_every_routing(report):
    assert report["bad_heavy"] == 0


def test_prefill_workspaces_are_bounded(report):
    # 8K and 32K tokens with H = 2048, I = 768, 512 experts, top-10 and a shared expert
    assert 0 < report["ws_8k"] < 4 << 30
    assert report["ws_8k"] < report["ws_32k"] < 12 << 30


def test_row_tiles_split_between_the_gemms(report):
    # every row tile in exactly one of the wide, mma.sync and dequantising
    # lists, and each list exercised by the sampled routings
    assert report["bad_split"] == 0
    assert report["n_wide"] > 0 and report["n_mma"] > 0 and report["n_light"] > 0
