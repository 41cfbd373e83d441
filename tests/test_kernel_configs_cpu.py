"""The GEMM kernel's compile-time configurations (GemmCfg), checked on the CPU.

A small host program built against csrc/dq_gemm.cuh prints every
configuration the library instantiates; the resource and ring invariants the
kernel relies on are asserted here, so that a change to the ring arithmetic
that would overflow shared or tensor memory, overrun a barrier array, or let
the next-tile preparation wait on itself fails before any GPU run."""

import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "weight_only_quantized_prologue_b200", "csrc")
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

# (format enum name, its value, tile heights the library instantiates)
INSTANCES = [
    ("FMT_INT4", 0, (16, 32, 64, 128, 256)), ("FMT_NVFP4", 1, (16, 32, 64, 128, 256)),
    ("FMT_MXFP4", 2, (16, 32, 64, 128, 256)), ("FMT_FP8", 3, (16, 32, 64, 128, 256)),
    ("FMT_FP8S", 4, (16, 32, 64, 128)), ("FMT_INT4A", 5, (16, 32, 64, 128, 256)),
    ("FMT_W4A4MX", 6, (32, 64, 128, 256)), ("FMT_W4A4NV", 7, (32, 64, 128, 256)),
    ("FMT_FP8SQ", 8, (16, 32, 64, 128, 256)), ("FMT_MLP", 9, (16, 32, 64)),
]

PROGRAM = r"""
#include "dq_gemm.cuh"
#include <cstdio>
using namespace dq;
template <int F, int BN> void pr(bool& first) {
  using C = GemmCfg<F, BN>;
  std::printf("%s{\"fmt\": %d, \"bn\": %d, \"smem\": %d, \"budget\": %d, \"tmem\": %d, \"a_cols\": %d, "
              "\"acc_col\": %d, \"acc_bufs\": %d, \"issuers\": %d, \"mlp\": %d, \"xst\": %d, \"wst\": %d, "
              "\"qst\": %d, \"a_stages\": %d, \"prefill\": %d, \"w4a4\": %d, \"ss\": %d, \"tsa\": %d, "
              "\"x_slot\": %d, \"w_slot\": %d, \"recv_off\": %d, \"bar_off\": %d, \"epi_off\": %d}",
              first ? "" : ",\n", F, BN, C::SMEM, C::SMEM_BUDGET, C::TMEM_COLS, C::A_COLS, C::ACC_COL,
              C::ACC_BUFS, C::ISSUERS, (int)C::MLP, C::XST, C::WST, C::QST, C::A_STAGES, C::PREFILL,
              (int)C::W4A4, (int)C::SS, (int)C::TSA, C::X_SLOT, C::W_SLOT, C::RECV_OFF, C::BAR_OFF, C::EPI_OFF);
  first = false;
}
int main() {
  bool first = true;
  std::printf("[");
@CALLS@
  std::printf("]\n");
}
"""


@pytest.fixture(scope="module")
def configs(tmp_path_factory):
    if not os.path.exists(NVCC):
        pytest.skip("nvcc not available")
    calls = "\n".join(f"  pr<{name}, {bn}>(first);" for name, _, bns in INSTANCES for bn in bns)
    d = tmp_path_factory.mktemp("cfg")
    src = d / "cfg.cu"
    src.write_text(PROGRAM.replace("@CALLS@", calls))
    exe = d / "cfg"
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "--expt-relaxed-constexpr",
                    "-I", CSRC, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return json.loads(out)


def test_every_instance_is_listed(configs):
    assert len(configs) == sum(len(bns) for _, _, bns in INSTANCES)


def test_shared_memory_fits(configs):
    for c in configs:
        assert c["smem"] <= 227 * 1024, c
        # the skinny budgets are sized so that two CTAs share an SM (the next
        # call's beside this one): 2 x (smem + 1 KB reserved) <= 228 KB.  The
        # one exception: the one-launch MLP's 64-row tile, which holds layer
        # 2's weight and operand and the split-K receive area besides its rings
        # and runs one CTA per SM
        if c["budget"] <= 108 * 1024 and not (c["mlp"] and c["bn"] == 64):
            assert 2 * (c["smem"] + 1024) <= 228 * 1024, c
        # the regions are laid out in order inside the allocation
        assert c["recv_off"] <= c["bar_off"] < c["epi_off"] < c["smem"], c


def test_tensor_memory_fits(configs):
    for c in configs:
        accs = (2 if c["mlp"] else c["acc_bufs"]) * c["issuers"] * c["bn"]
        assert c["acc_col"] == c["a_cols"], c
        assert c["a_cols"] + accs <= c["tmem"] <= 512, c
        assert c["tmem"] in (32, 64, 128, 256, 512), c
        if c["budget"] <= 108 * 1024:        # two CTAs per SM share its 512 columns
            assert c["tmem"] <= 256, c


def test_rings_fit_their_barrier_arrays(configs):
    for c in configs:
        assert 2 <= c["xst"] <= 8 and 2 <= c["wst"] <= 8 and 0 <= c["a_stages"] <= 8 and c["qst"] <= 8, c
        if c["tsa"] and c["fmt"] == 4:        # fused static FP8: bf16 and operand rings
            assert c["qst"] >= 2, c


def test_next_tile_preparation_cannot_wait_on_itself(configs):
    # the prologue warps prepare up to PREFILL stages of a persistent CTA's
    # next tile before this tile's epilogue; where only MMAs (which wait for
    # that epilogue) free the weight and x slots, PREFILL must not exceed them
    for c in configs:
        assert c["prefill"] <= c["a_stages"], c
        if c["w4a4"]:
            assert c["prefill"] <= min(c["xst"], c["wst"]), c


def test_double_buffered_accumulator_only_where_the_epilogue_warps_are_free(configs):
    # two accumulators only for static FP8 on e4m3 codes at 256-row tiles,
    # whose epilogue warps have no per-stage work
    for c in configs:
        if c["acc_bufs"] == 2:
            assert c["fmt"] == 8 and c["bn"] == 256 and c["ss"] and c["a_cols"] == 0, c
