"""DRAM traffic per launch (ncu `dram__bytes_read.sum + dram__bytes_write.sum`)
of the library's kernels, stamped with a digest of the sources they were
built from, so that a kernel change turns every recorded figure stale.

Record (after captures of the launch list with those two metrics, one pass):

    python -m tiled_attention_24_b200.traffic \\
        fwd_bf16_prefill_noncausal=fwd_traffic.csv:0 \\
        decode_split=decode_traffic.csv:0:8 ...

Each argument is KEY=CSV:ID[:SCALE]: the launch with that ID in an ncu
`--csv` log, its read + write bytes times SCALE (a smaller capture scaled to
the full launch by the units it processes).  The file is rewritten with the
current digest and only the entries given.

`load()` returns the entries whose digest matches the sources as they are
now, and nothing otherwise.
"""
from __future__ import annotations

import csv
import hashlib
import json
import os
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
PATH = os.path.join(ROOT, "profiles", "traffic.json")
_LIB_SOURCES = ("csrc", ("api.cu", "bwd_bf16.cuh", "decode.cuh", "decode_tc.cuh", "exp2_poly.cuh", "fwd_bf16.cuh",
                         "fwd_fp4.cuh", "fwd_fp8.cuh", "fwd_int8.cuh", "ptx.cuh", "quant.cuh"))


def library_digest() -> str:
    """sha256 (first 16 hex digits) over the kernel and launch sources of
    libtiledattn.so and its header, in a fixed order."""
    h = hashlib.sha256()
    files = [os.path.join(PKG, _LIB_SOURCES[0], f) for f in _LIB_SOURCES[1]]
    files.append(os.path.join(ROOT, "include", "tiledattn.h"))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load(path: str = PATH) -> dict:
    """{key: bytes per launch} if the file's digest matches the sources, else {}."""
    try:
        with open(path) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return {}
    if data.get("sources") != library_digest():
        return {}
    return {k: v for k, v in data.get("bytes_per_launch", {}).items()}


def launch_bytes(csv_path: str, launch_id: int) -> int:
    """read + write DRAM bytes of one launch of an ncu --csv log."""
    with open(csv_path) as f:
        rows = [r for r in csv.reader(line for line in f if line.startswith('"'))]
    head, body = rows[0], rows[1:]
    iid, iname, ival = head.index("ID"), head.index("Metric Name"), head.index("Metric Value")
    got = {}
    for r in body:
        if int(r[iid]) == launch_id and r[iname] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            got[r[iname]] = float(r[ival].replace(",", ""))
    if len(got) != 2:
        raise ValueError(f"{csv_path}: launch {launch_id} lacks the two dram byte metrics")
    return int(sum(got.values()))


def main(argv) -> int:
    out = {}
    for a in argv:
        key, spec = a.split("=", 1)
        parts = spec.split(":")
        scale = float(parts[2]) if len(parts) > 2 else 1.0
        out[key] = int(round(launch_bytes(parts[0], int(parts[1])) * scale))
    data = {"_what": "dram__bytes_read.sum + dram__bytes_write.sum per launch from ncu; valid only while "
                     "'sources' equals the digest of the library's kernel sources",
            "sources": library_digest(), "bytes_per_launch": out}
    with open(PATH, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    print(json.dumps(data, indent=1))
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
