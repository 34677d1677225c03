"""Reader of tests/golden/index_order_cases.txt: builds the byte arrays of the
hand-worked index-score and indexer-K cases.  It only places codes and scale
bytes where the file says; it computes nothing of the method."""
import os

import numpy as np

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "index_order_cases.txt")
UNIT_SCALE = 0x38  # E4M3 1.0: the scale byte of every block the file does not list


def _chan_range(s):
    a, b = s.split("-")
    return int(a), int(b)


def _put_codes(codes, c0, c1, code):
    """codes: u8 [32] packed E2M1 (channel 2j low nibble of byte j, 2j+1 high)."""
    for c in range(c0, c1 + 1):
        j = c // 2
        if c % 2 == 0:
            codes[j] = (codes[j] & 0xF0) | code
        else:
            codes[j] = (codes[j] & 0x0F) | (code << 4)


def load():
    """-> (score_cases, kproj_cases).  A score case is a dict with q [128] u8,
    qs [16] u8, w [4] f32 and entries: list of dicts (pos, k [32], ks [4], score),
    plus top1.  A kproj case has x [512] f32 values, W [512, 64] f32, out {j: v},
    kcodes [8] and kscale0."""
    score_cases, kproj_cases = [], []
    cur = None
    with open(PATH, encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            op = tok[0]
            if op == "case":
                name = tok[1]
                if name.startswith("kproj"):
                    cur = dict(kind="kproj", name=name, x=np.zeros(512, np.float32),
                               W=np.zeros((512, 64), np.float32), out={})
                else:
                    cur = dict(kind="score", name=name, q=np.zeros(128, np.uint8),
                               qs=np.full(16, UNIT_SCALE, np.uint8), w=np.zeros(4, np.float32), entries=[])
            elif op == "end":
                (kproj_cases if cur["kind"] == "kproj" else score_cases).append(cur)
                cur = None
            elif op == "w":
                cur["w"] = np.array([float.fromhex(t) for t in tok[1:5]], np.float32)
            elif op == "sq":
                h = int(tok[1])
                cur["qs"][4 * h:4 * h + 4] = [int(t, 16) for t in tok[2:6]]
            elif op == "q":
                h = int(tok[1])
                c0, c1 = _chan_range(tok[2])
                view = cur["q"][32 * h:32 * h + 32]
                _put_codes(view, c0, c1, int(tok[3]))
            elif op == "entry":
                cur["entries"].append(dict(pos=int(tok[1]), k=np.zeros(32, np.uint8),
                                           ks=np.full(4, UNIT_SCALE, np.uint8), score=None))
            elif op == "sk":
                cur["entries"][-1]["ks"][:] = [int(t, 16) for t in tok[1:5]]
            elif op == "k":
                c0, c1 = _chan_range(tok[1])
                _put_codes(cur["entries"][-1]["k"], c0, c1, int(tok[2]))
            elif op == "score":
                cur["entries"][-1]["score"] = np.float32(float.fromhex(tok[1]))
            elif op == "top1":
                cur["top1"] = int(tok[1])
            elif op == "x":
                cur["x"][int(tok[1])] = float.fromhex(tok[2])
            elif op == "W":
                cur["W"][int(tok[1]), int(tok[2])] = float.fromhex(tok[3])
            elif op == "out":
                cur["out"][int(tok[1])] = np.float32(float.fromhex(tok[2]))
            elif op == "kcodes":
                cur["kcodes"] = np.array([int(t, 16) for t in tok[1:]], np.uint8)
            elif op == "kscale0":
                cur["kscale0"] = int(tok[1], 16)
            else:
                raise ValueError(f"unknown line in {PATH}: {raw!r}")
    return score_cases, kproj_cases


def bf16_bits_of(values):
    """uint16 bf16 patterns of float32 values that are exact in bf16 (asserted)."""
    v = np.asarray(values, np.float32)
    u = v.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def keys_array(case, n, stride=1):
    """Row-major key codes [n, 32] and scales [n, 4] with the case's entries at
    position pos * stride (every other entry all-zero codes, unit scales).  A
    stride keeps the entries' order, so the tie rule decides the same way."""
    k = np.zeros((n, 32), np.uint8)
    ks = np.full((n, 4), UNIT_SCALE, np.uint8)
    for e in case["entries"]:
        k[e["pos"] * stride] = e["k"]
        ks[e["pos"] * stride] = e["ks"]
    return k, ks
