"""The end-to-end loop bench.py times computes the right thing (GPU).

bench.run_e2e is the public-API serving loop: the library's pool appends a
token to every sequence and packs the tables, the step's inputs cross to the
device from pinned memory, copy-on-write + append + decode run, and the output
comes back.  Here the loop runs a few steps on small variants of the decode
workloads and the last step's output is checked, on sampled sequences,
against the oracle over the caches and tables that step used.
"""
import argparse

import numpy as np
import pytest
import torch

import bench
import oracle
import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2, "fp8_e4m3": 3e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield


CASES = [
    ("llama3_8b_gqa_bf16_b128", 12, 300, 1200, None, 256),
    ("llama2_7b_mha_fp16_b64", 6, 100, 700, None, 0),
    ("prefix_shared_fp8_b256", 24, 10, 200, 256, 0),
]


@pytest.mark.parametrize("name,nseq,lo,hi,prefix,part", CASES, ids=[c[0] for c in CASES])
def test_e2e_loop_output_matches_the_oracle(name, nseq, lo, hi, prefix, part):
    cfg = wl.small_variant(wl.DECODE_WORKLOADS[name], nseq, lo, hi, prefix_tokens=prefix)
    args = argparse.Namespace(seed=4, warmup=3, steps=4, no_shared_prefix=False)
    r = bench.run_e2e(args, cfg, pa, torch.device("cuda", 0), part, keep_state=True)
    assert pa.pa_device_status() == 0
    st = r["state"]
    seqs = [0, nseq // 2, nseq - 1]
    want = oracle.paged_decode(st["q"], cfg.q_dtype, st["key_cache"], st["value_cache"],
                               cfg.kv_dtype, st["tables"], st["lens"], st["scale"],
                               st["k_scale"], st["v_scale"], seqs=seqs)
    got = st["out"][seqs].to(torch.float64).numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - want).max()
    assert err <= TOL[cfg.kv_dtype], f"{name}: max abs error {err:.3g}"
    # the loop grew every sequence by one token a step
    assert int(st["lens"].min()) >= lo + args.warmup + args.steps - 1
