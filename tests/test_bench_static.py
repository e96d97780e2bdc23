"""Host-side guards that need no GPU.

* bench.py builds its timed step from lambdas that look their tensors up when
  they run; a name such a lambda reads must not be rebound later in the same
  function (a later block reusing it would hand the kernel another tensor).
* the binding rejects buffers whose shape or dtype does not match the call
  before anything reaches the C ABI.
"""
import ast
import json
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _assigned_names(fn):
    counts = {}
    for node in ast.walk(fn):
        targets = []
        if isinstance(node, ast.Assign):
            targets = node.targets
        elif isinstance(node, (ast.AugAssign, ast.AnnAssign)):
            targets = [node.target]
        elif isinstance(node, (ast.For, ast.comprehension)):
            targets = [node.target]
        for t in targets:
            for n in ast.walk(t):
                if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Store):
                    counts[n.id] = counts.get(n.id, 0) + 1
    return counts


def _lambda_free_names(lam):
    params = {a.arg for a in lam.args.args + lam.args.kwonlyargs}
    return {n.id for n in ast.walk(lam.body) if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)} - params


def test_bench_step_lambdas_read_names_bound_once():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    fn = next(n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef) and n.name == "run_ours")
    counts = _assigned_names(fn)
    bad = set()
    for lam in (n for n in ast.walk(fn) if isinstance(n, ast.Lambda)):
        for name in _lambda_free_names(lam):
            if counts.get(name, 0) > 1:
                bad.add(name)
    assert not bad, f"names read by step lambdas and assigned more than once: {sorted(bad)}"


def test_binding_rejects_mis_shaped_buffers():
    from tiled_attention_24_b200 import _binding as b
    ok = torch.empty(2, 3, 4, dtype=torch.bfloat16)
    b._expect((ok, (2, 3, 4), torch.bfloat16, "x"))
    with pytest.raises(ValueError):
        b._expect((ok, (2, 3, 5), torch.bfloat16, "x"))
    with pytest.raises(ValueError):
        b._expect((ok, (2, 3, 4), torch.float32, "x"))
    with pytest.raises(ValueError):
        b._at_least(torch.empty(10, dtype=torch.uint8), 11, "codes")


def test_traffic_record_is_dropped_when_the_sources_change(tmp_path, monkeypatch):
    """profiles/traffic.json holds ncu DRAM bytes stamped with a digest of the
    kernel sources; a record from other sources reads as empty."""
    from tiled_attention_24_b200 import traffic
    log = tmp_path / "t.csv"
    log.write_text(
        "==PROF== Connected to process 1\n"
        '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
        '"0","k","dram__bytes_read.sum","byte","1,000"\n'
        '"0","k","dram__bytes_write.sum","byte","24"\n'
        '"1","k","dram__bytes_read.sum","byte","7"\n'
        '"1","k","dram__bytes_write.sum","byte","1"\n')
    assert traffic.launch_bytes(str(log), 0) == 1024 and traffic.launch_bytes(str(log), 1) == 8
    out = tmp_path / "traffic.json"
    monkeypatch.setattr(traffic, "PATH", str(out))
    traffic.main([f"a={log}:0", f"b={log}:1:8"])
    assert traffic.load(str(out)) == {"a": 1024, "b": 64}
    data = json.loads(out.read_text())
    data["sources"] = "0" * 16
    out.write_text(json.dumps(data))
    assert traffic.load(str(out)) == {}


def test_traffic_digest_covers_every_kernel_source():
    """Every source file libtiledattn.so is compiled from (api.cu and the
    headers it includes) is part of the digest, so that no kernel can change
    under a stale traffic record."""
    import re
    from tiled_attention_24_b200 import traffic
    csrc = os.path.join(traffic.PKG, traffic._LIB_SOURCES[0])
    seen, todo = set(), ["api.cu"]
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.add(f)
        with open(os.path.join(csrc, f)) as fh:
            todo += [m for m in re.findall(r'#include "([^"]+)"', fh.read()) if os.path.exists(os.path.join(csrc, m))]
    assert seen <= set(traffic._LIB_SOURCES[1]), sorted(seen - set(traffic._LIB_SOURCES[1]))
