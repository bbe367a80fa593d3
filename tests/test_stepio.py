"""A step written by stepio (the format bench.py --dump uses) reads back
unchanged, and replaying its inputs through the oracle reproduces the stored
outputs: the path a user takes to check a step seen on the GPU elsewhere."""
import numpy as np

import oracle
from ddtree_speculative_decode_b200 import stepio, synth


def _step():
    s = synth.custom(B=2, D=4, K=3, N=16, H=2, d_l=32, d_r=8, V=300, L=(20, 7), dtype="bf16", seed=5,
                     accept_p=0.9)
    x = synth.make_step(s)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    logits = synth.target_logits(s, tree["parent"], tree["node_tok"], tree["n_nodes"])
    return s, x, tree, logits


def _outputs(s, x, tree, logits):
    out, lse = oracle.verify_attn(x.q, x.kv, x.cache_off, x.cache_len, tree["mask"], tree["n_nodes"], s.H, s.d_l,
                                  s.d_r, s.scale, s.dtype)
    kv = x.kv.copy()
    acc = oracle.accept_compact(logits, s.dtype, tree["node_tok"], tree["parent"], tree["n_nodes"], kv,
                                x.cache_off, x.cache_len, x.cache_cap)
    o = {k: v for k, v in tree.items()}
    o.update({f"acc_{k}": v for k, v in acc.items() if k != "cache_len"})
    o["attn_out"] = out.astype(np.float32)
    o["lse"] = lse.astype(np.float32)
    o["cache_len_after"] = acc["cache_len"]
    return o


def test_round_trip(tmp_path):
    s, x, tree, logits = _step()
    inputs = {"logp": x.logp, "tok": x.tok, "root_tok": x.root_tok, "cache_len": x.cache_len,
              "cache_off": x.cache_off, "cache_cap": x.cache_cap, "q": x.q, "kv": x.kv, "logits": logits}
    outputs = _outputs(s, x, tree, logits)
    meta = {"workload": s.name, "N": s.N, "H": s.H, "d_latent": s.d_l, "d_rope": s.d_r, "dtype": s.dtype,
            "scale": s.scale}
    path = str(tmp_path / "step.npz")
    stepio.save_step(path, inputs, outputs, meta)
    i2, o2, m2 = stepio.load_step(path)
    assert m2 == meta
    assert set(i2) == set(inputs) and set(o2) == set(outputs)
    for k, v in inputs.items():
        assert i2[k].dtype == np.asarray(v).dtype and np.array_equal(i2[k], v), k
    for k, v in outputs.items():
        assert np.array_equal(o2[k], v, equal_nan=True), k


def test_replay_through_the_oracle(tmp_path):
    s, x, tree, logits = _step()
    inputs = {"logp": x.logp, "tok": x.tok, "root_tok": x.root_tok, "cache_len": x.cache_len,
              "cache_off": x.cache_off, "cache_cap": x.cache_cap, "q": x.q, "kv": x.kv, "logits": logits}
    path = str(tmp_path / "step.npz")
    stepio.save_step(path, inputs, _outputs(s, x, tree, logits),
                     {"N": s.N, "H": s.H, "d_latent": s.d_l, "d_rope": s.d_r, "dtype": s.dtype, "scale": s.scale})
    i, o, m = stepio.load_step(path)
    t = oracle.build_tree(i["logp"], i["tok"], i["root_tok"], i["cache_len"], m["N"])
    for k in ("node_tok", "parent", "depth", "pos", "n_nodes", "mask"):
        assert np.array_equal(t[k], o[k]), k
    out, _ = oracle.verify_attn(i["q"], i["kv"], i["cache_off"], i["cache_len"], o["mask"], o["n_nodes"], m["H"],
                                m["d_latent"], m["d_rope"], m["scale"], m["dtype"])
    assert np.abs(out - o["attn_out"]).max() <= 1e-6 * max(1.0, np.abs(out).max())
    kv = i["kv"].copy()
    acc = oracle.accept_compact(i["logits"], m["dtype"], o["node_tok"], o["parent"], o["n_nodes"], kv,
                                i["cache_off"], i["cache_len"], i["cache_cap"])
    for k in ("acc_len", "acc_nodes", "out_tok", "bonus", "am"):
        assert np.array_equal(acc[k], o[f"acc_{k}"]), k
    assert np.array_equal(acc["cache_len"], o["cache_len_after"])
