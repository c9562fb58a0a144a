"""Writes the oracle's AWQ search over one LLaMA-2-7B-shaped decoder block
(the four search places of "MIT 6.5940 Lab 4 + Lab 5", "Question 2", mapped
to q|k|v, o, gate|up and down; synthetic calibration input T = 512, 1 %
outlier channels x20; 20 alphas; group 128) for the GPU parity test, which
would otherwise spend minutes recomputing it on the host.

Calls only ``oracle`` and ``synth``. Stored per place: the 20 fp64 losses
(as exact hex floats), the chosen index, and SHA-256 digests of the fp64
activation means and of the chosen fp16 scales (bit-exact checks).

    python tests/golden/make_awq_block_golden.py [bits ...]    (default: 4 3)
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle as O  # noqa: E402
import synth  # noqa: E402


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def main(bits_list):
    for bits in bits_list:
        out = {"source": "oracle.awq_search over synth.config_awq_block(5): one LLaMA-2-7B-shaped block, "
                         f"T=512, 20 alphas j/20, {bits}-bit asymmetric, group 128",
               "bits": bits, "group": 128, "symmetric": False, "places": {}}
        for name, X, named in synth.config_awq_block(5):
            r = O.awq_search(X, [W for _, W in named], bits, 128, False)
            L = r["losses"]
            order = np.argsort(L, kind="stable")
            out["places"][name] = {
                "T": int(X.shape[0]), "K": int(X.shape[1]), "N": [int(W.shape[0]) for _, W in named],
                "losses_hex": [float(v).hex() for v in L],
                "best": int(r["best"]),
                "gap12": float((L[order[1]] - L[order[0]]) / L[order[0]]),
                "mu_sha256": digest(r["mu"]),
                "s_sha256": digest(r["s"].view(np.uint16)),
            }
            print(bits, name, out["places"][name]["best"], out["places"][name]["gap12"], flush=True)
        with open(os.path.join(HERE, f"awq_llama7b_block_w{bits}_oracle.json"), "w") as f:
            json.dump(out, f, indent=1)


if __name__ == "__main__":
    main([int(b) for b in sys.argv[1:]] or [4, 3])
