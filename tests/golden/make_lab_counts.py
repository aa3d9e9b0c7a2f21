"""Write lab_counts.json: the lab's count tables at the lab's model sizes.

Calls only ``oracle.lab``.  The sizes are those of TT Lab
"キー・バリューヘッドだけ減らしてみる", step 8 ("何が減り、何が減らないのかを記録する"):
layers=32, seq_len=4096, head_dim=128, h=8, d_model=1024, n_tokens=4096,
groups [8, 4, 2, 1].  The page prints the sizes and the formulas (steps 6-7)
but no resulting numbers; the stored numbers are the oracle's.

Run from the repository root:  python tests/golden/make_lab_counts.py
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import lab  # noqa: E402

LAYERS, SEQ_LEN, HEAD_DIM, H, D_MODEL, N_TOKENS = 32, 4096, 128, 8, 1024, 4096
GROUPS = [8, 4, 2, 1]


def main():
    kv = lab.kv_table(LAYERS, H, GROUPS, SEQ_LEN, HEAD_DIM)
    mults = {g: lab.mults(N_TOKENS, D_MODEL, H, g, HEAD_DIM) for g in GROUPS}
    out = {
        "source": "TT Lab tf-gqa-lab step 8 sizes; formulas of steps 6-7",
        "sizes": {"layers": LAYERS, "seq_len": SEQ_LEN, "head_dim": HEAD_DIM, "h": H,
                  "d_model": D_MODEL, "n_tokens": N_TOKENS, "groups": GROUPS},
        "kv_table": [[g, n] for g, n in kv],
        "mult_table": {str(g): mults[g] for g in GROUPS},
    }
    path = os.path.join(HERE, "lab_counts.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
