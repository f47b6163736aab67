"""The algorithmic byte counts behind the benchmark's GB/s and roofline
fractions, checked on the CPU against the storage format and hand-worked
figures.

* Quantised draft: a layer call must read every group record of every (request,
  KV head) once, plus the bf16 residual K and V; the record size comes from the
  cache format (oracle/quant.py, record_layout), independently of the bench's
  own per-part formula.
* Verification: the full bf16 K and V of the layer.
* Token-dropped draft: the kept K and V rows and their int32 positions.
"""

import pytest

import bench
from oracle import quant as Q

QUANT = [k for k, w in bench.WORKLOADS.items() if "bits" in w]


@pytest.mark.parametrize("name", QUANT)
def test_quant_draft_bytes_match_the_record_format(name):
    w = bench.WORKLOADS[name]
    groups = (w["T"] - w["R"]) // w["G"]
    assert groups * w["G"] == w["T"] - w["R"], "the quantised span is whole groups"
    rec = Q.record_layout(w["bits"], w["G"], w["D"])["size"]
    per_unit = groups * rec + 2 * w["R"] * w["D"] * 2
    assert bench.draft_bytes_per_layer(w) == per_unit * w["B"] * w["Hkv"]


def test_llama_8b_layer_figures_by_hand():
    w = bench.WORKLOADS["llama-3.1-8b-32k-kivi2"]
    # per (request, head): 32640 quantised tokens -> 1020 records of 2*1024 + 8*128 = 3072 B,
    # plus 128 residual rows of bf16 K and V (128 * 128 * 4 B)
    assert bench.draft_bytes_per_layer(w) == 64 * (1020 * 3072 + 65536) == 204_734_464
    # verification: 8 requests x 8 heads x 32768 keys x 128 channels x (K + V) x 2 B
    assert bench.verify_bytes_per_layer(w) == 8 * 8 * 32768 * 128 * 4 == 1_073_741_824


def test_token_dropped_layer_figure_by_hand():
    w = bench.WORKLOADS["qwen-32b-100k-tokdrop4-streamed"]
    # 8 heads x 25000 kept rows x (256 B of K + 256 B of V + a 4-byte position)
    assert bench.sparse_bytes_per_layer(w) == 8 * 25000 * 516 == 103_200_000


def test_500k_and_70b_figures_by_hand():
    w5 = bench.WORKLOADS["llama-3.1-8b-1m-500k-kivi2"]
    # 499872 quantised tokens = 15621 records of 3072 B, plus the residual, per head
    assert bench.draft_bytes_per_layer(w5) == 8 * (15621 * 3072 + 65536) == 384_425_984
    w4 = bench.WORKLOADS["llama-70b-4x131k-4bit-stagger"]
    # 4-bit group 64: a record is 2 * 64*128*4/8 + 8*128 = 9216 B for 64 tokens; 2046 records per head
    assert Q.record_layout(4, 64, 128)["size"] == 9216
    assert bench.draft_bytes_per_layer(w4) == 8 * (2046 * 9216 + 65536)
