"""The decode step captured in a CUDA graph (GPU).

A serving loop launches the same decode step over and over; capturing it once
in a CUDA graph and replaying it takes the host's launch work off the step.
Every entry point of the step enqueues only kernels on the caller's stream
(no allocation, no synchronisation, no host read of device memory), so the
step can be captured.  Here the append + copy-on-write and the decode are
captured, the inputs are changed in place, and the replayed outputs must be
bit-identical to the eagerly launched calls on the same inputs.  The
shared-prefix step is replayed with both suffix passes (one CTA per suffix,
and the persistent grid, whose whole items wait for the prefix kernel only
before they fold its records); the prefill step (append + pa_prefill) too.
"""
import pytest
import torch

import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield


CASES = [
    ("llama3_8b_gqa_bf16_b128", 16, 300, 3000, None, 512, pa.DECODE_DEFAULT),
    ("long_context_splitk_bf16_4x100k", 2, 20000, 30000, None, 512, pa.DECODE_DEFAULT),
    ("prefix_shared_fp8_b256", 48, 10, 400, 512, 0, pa.DECODE_DEFAULT),
    ("prefix_shared_fp8_b256", 300, 10, 400, 512, 0,
     pa.DECODE_DEFAULT | pa.DECODE_SUFFIX_PERSISTENT),
]


@pytest.fixture
def select():
    yield pa.pa_decode_select
    pa.pa_decode_select(pa.DECODE_DEFAULT)


@pytest.mark.parametrize("name,nseq,lo,hi,prefix,part,mode", CASES,
                         ids=[c[0] + ("_persistent" if c[6] & pa.DECODE_SUFFIX_PERSISTENT else "")
                              for c in CASES])
def test_graph_replay_matches_eager_calls(name, nseq, lo, hi, prefix, part, mode, select):
    select(mode)
    cfg = wl.small_variant(wl.DECODE_WORKLOADS[name], nseq, lo, hi, prefix_tokens=prefix)
    inp = wl.make_decode_inputs(cfg, seed=21, device="cuda")
    S, Hq, D = inp.q.shape
    max_ctx = int(inp.context_lens.max())
    if prefix:
        ws_bytes = pa.pa_decode_shared_prefix_workspace_size(
            S, Hq, cfg.num_kv_heads, D, cfg.block_size, max_ctx, prefix, inp.key_cache.dtype)
    else:
        ws_bytes = pa.pa_decode_workspace_size(S, Hq, D, max_ctx, part)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    kc, vc = inp.key_cache.clone(), inp.value_cache.clone()
    q, kn, vn = inp.q.clone(), inp.key_new.clone(), inp.value_new.clone()
    out = torch.empty_like(q)

    def append():
        if inp.copy_pairs.numel():
            pa.pa_copy_blocks(kc, vc, inp.copy_pairs)
        pa.pa_reshape_and_cache(kn, vn, kc, vc, inp.slot_mapping, inp.k_scale, inp.v_scale)

    def decode():
        if prefix:
            pa.pa_decode_shared_prefix(out, q, kc, vc, inp.block_tables, inp.context_lens,
                                       max_ctx, inp.scale, prefix, ws, inp.k_scale, inp.v_scale)
        else:
            pa.pa_decode(out, q, kc, vc, inp.block_tables, inp.context_lens, max_ctx, inp.scale,
                         inp.k_scale, inp.v_scale, part, ws)

    append()
    decode()
    torch.cuda.synchronize()
    g_app, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app):
        append()
    with torch.cuda.graph(g_dec):
        decode()
    gen = torch.Generator(device="cuda").manual_seed(5)
    for _ in range(3):
        # new inputs in place: the graphs read them from the same addresses
        q.copy_(torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype))
        kn.copy_(torch.randn(kn.shape, generator=gen, device="cuda").to(kn.dtype))
        vn.copy_(torch.randn(vn.shape, generator=gen, device="cuda").to(vn.dtype))
        g_app.replay()
        g_dec.replay()
        torch.cuda.synchronize()
        got, kc_g, vc_g = out.clone(), kc.clone(), vc.clone()
        append()
        decode()
        torch.cuda.synchronize()
        assert pa.pa_device_status() == 0
        assert torch.equal(wl.raw_view(kc_g, cfg.kv_dtype), wl.raw_view(kc, cfg.kv_dtype))
        assert torch.equal(wl.raw_view(vc_g, cfg.kv_dtype), wl.raw_view(vc, cfg.kv_dtype))
        assert torch.isfinite(got).all()
        assert torch.equal(got, out), "graph replay differs from the eager calls"


def test_prefill_graph_replay_matches_eager_calls():
    cfg = wl.PrefillConfig("graph", 3, 32, 8, 128, 16, "bf16", 100, 700, 0, 900)
    inp = wl.make_prefill_inputs(cfg, seed=22)
    d = {k: getattr(inp, k).cuda() for k in ("q", "key_cache", "value_cache", "key_new",
                                              "value_new", "slot_mapping", "block_tables",
                                              "context_lens", "query_start")}
    kc, vc = d["key_cache"].clone(), d["value_cache"].clone()
    out = torch.empty_like(d["q"])

    def step():
        pa.pa_reshape_and_cache(d["key_new"], d["value_new"], kc, vc, d["slot_mapping"])
        pa.pa_prefill(out, d["q"], kc, vc, d["block_tables"], d["context_lens"], d["query_start"],
                      inp.max_query_len, inp.scale)

    step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    gen = torch.Generator(device="cuda").manual_seed(6)
    for _ in range(3):
        for k in ("q", "key_new", "value_new"):
            d[k].copy_(torch.randn(d[k].shape, generator=gen, device="cuda").to(d[k].dtype))
        g.replay()
        torch.cuda.synchronize()
        got, kc_g = out.clone(), kc.clone()
        step()
        torch.cuda.synchronize()
        assert pa.pa_device_status() == 0
        assert torch.equal(wl.raw_view(kc_g, cfg.dtype), wl.raw_view(kc, cfg.dtype))   # NaN-poisoned slots
        assert torch.isfinite(got).all()
        assert torch.equal(got, out), "graph replay differs from the eager calls"
