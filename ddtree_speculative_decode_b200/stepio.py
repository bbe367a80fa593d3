"""One verify step's inputs and outputs written to (and read back from) a
compressed .npz file, so a step seen on the GPU can be replayed elsewhere
(another build of the library, or a CPU check).

Arrays keep their stored form: bf16 tensors as uint16 bit patterns, float32
as float32, integers as they are. Keys are prefixed "in/" and "out/"; "meta"
holds a JSON string (workload name, sizes, dtype)."""
from __future__ import annotations

import json

import numpy as np


def save_step(path: str, inputs: dict, outputs: dict, meta: dict) -> None:
    arrays = {f"in/{k}": np.ascontiguousarray(v) for k, v in inputs.items()}
    arrays.update({f"out/{k}": np.ascontiguousarray(v) for k, v in outputs.items()})
    arrays["meta"] = np.array(json.dumps(meta))
    np.savez_compressed(path, **arrays)


def load_step(path: str):
    """Returns (inputs, outputs, meta) as written by save_step."""
    with np.load(path, allow_pickle=False) as z:
        inputs = {k[3:]: z[k] for k in z.files if k.startswith("in/")}
        outputs = {k[4:]: z[k] for k in z.files if k.startswith("out/")}
        meta = json.loads(str(z["meta"]))
    return inputs, outputs, meta
