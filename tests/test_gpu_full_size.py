"""GPU parity at the workloads' full sizes, through the C-ABI binding.

* The 64K-context case (B1 Hq64 Hkv8, 65,536 tokens, 0.1 % outliers) and the
  128K-context case (B1 Hq96 Hkv8, 131,072 tokens, GQA group 12, prefilled by
  2048-token chunked appends) compare every output row with the fp64 oracle.
* The benchmark's own steps -- its DecodeWorkload, replicas and launch
  sequence (append one token per sequence, then attention) -- for the ragged
  B128 workload (sampled sequences, computed one by one by the oracle) and
  for the 4K GQA decode step (every sequence).

Tolerance: max-abs 2e-2 and mean-abs 2e-3 against the oracle over the same
FP8 values.  Inputs come only from `synthetic` (through bench.py's block
generator for the benchmark workloads); expected values only from `oracle`.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import synthetic
from cases import Case, assert_attention_close

pytestmark = pytest.mark.gpu


def test_long64k_full_size():
    c = Case(synthetic.get("long64k"))
    got = c.gpu_attention().cpu().numpy()
    assert c.status.item() == 0
    assert_attention_close(got, c.oracle_attention())


def test_moe128k_full_size_group12_chunked():
    c = Case(synthetic.get("moe128k"), prefill_chunk=2048)
    got = c.gpu_attention().cpu().numpy()
    assert c.status.item() == 0
    assert_attention_close(got, c.oracle_attention())


def _oracle_tensor_scale(w, L_max, which, replicas):
    """fl32(amax / 2688) over every token the benchmark calibrates on: the
    prefill blocks (all L_max slots of every sequence) and the replicas' new
    tokens.  The scale is monotone in amax, so the largest block scale is the
    scale of the whole tensor."""
    scales = []
    for c in range((w.B + bench.GEN_SEQS - 1) // bench.GEN_SEQS):
        x = bench.gen_block(w, L_max, which, c).numpy()
        rc, s = oracle.tensor_scale(x.ravel())
        assert rc == 0
        scales.append(s)
        del x
    rc, s = oracle.tensor_scale(synthetic.kv_tokens(w, replicas, which, stream=1).numpy().ravel())
    assert rc == 0
    scales.append(s)
    return np.float32(max(scales))


def _oracle_step(w, L_max, b, L, sk, sv, replica=0, replicas=2):
    """The oracle's output rows for sequence b after one benchmark step on
    replica `replica`: its L cached tokens, the new token at slot L, fp64
    attention over L + 1 tokens."""
    c, i = divmod(b, bench.GEN_SEQS)
    xk = bench.gen_block(w, L_max, "k", c)[i:i + 1, :L].numpy()
    xv = bench.gen_block(w, L_max, "v", c)[i:i + 1, :L].numpy()
    nk = synthetic.kv_tokens(w, replicas, "k", stream=1)[b:b + 1, replica:replica + 1].numpy()
    nv = synthetic.kv_tokens(w, replicas, "v", stream=1)[b:b + 1, replica:replica + 1].numpy()
    q = synthetic.queries(w, stream=replica)[b:b + 1].numpy()
    S = synthetic.capacity(L + 1)
    kc, ks = oracle.new_planes(1, w.Hkv, S, w.D)
    vc, vs = oracle.new_planes(1, w.Hkv, S, w.D)
    z = np.zeros(1, np.int32)
    at = np.array([L], np.int32)
    assert oracle.quantize_append(xk, z, sk, kc, ks) == 0
    assert oracle.quantize_append(xv, z, sv, vc, vs) == 0
    assert oracle.quantize_append(nk, at, sk, kc, ks) == 0
    assert oracle.quantize_append(nv, at, sv, vc, vs) == 0
    return oracle.decode_attention_nvfp4(q, kc, ks, vc, vs, sk, sv, np.array([L + 1], np.int32))[0]


def _bench_step_check(name, sample):
    w = synthetic.get(name)
    R = 2
    wl = bench.DecodeWorkload(w, R, with_append=True)
    wl.step(0)
    torch.cuda.synchronize()
    assert wl.status.item() == 0
    got = wl.out[0].cpu().numpy()
    L_max = max(wl.lens0)
    sk = _oracle_tensor_scale(w, L_max, "k", R)
    sv = _oracle_tensor_scale(w, L_max, "v", R)
    # the device calibrated on the same tokens: the scales agree bit for bit
    assert np.float32(wl.sk.item()).view(np.uint32) == sk.view(np.uint32)
    assert np.float32(wl.sv.item()).view(np.uint32) == sv.view(np.uint32)
    bs = sample(wl.lens0)
    want = np.stack([_oracle_step(w, L_max, b, wl.lens0[b], sk, sv, replicas=R) for b in bs])
    assert_attention_close(got[bs], want)
    del wl
    torch.cuda.empty_cache()


def test_bench_ragged_step_matches_oracle():
    """The headline workload: B128, lengths U[1024, 8192]; the shortest, the
    longest and six seeded sequences in between."""
    def sample(lens):
        order = np.argsort(lens)
        rng = np.random.default_rng(11)
        mid = rng.choice(order[1:-1], size=6, replace=False)
        return [int(order[0]), int(order[-1])] + [int(b) for b in mid]
    _bench_step_check("ragged", sample)


def test_bench_gqa_step_matches_oracle():
    """The 4K GQA decode step (B8, 4096 cached tokens + 1 appended): every sequence."""
    _bench_step_check("gqa", lambda lens: list(range(len(lens))))
