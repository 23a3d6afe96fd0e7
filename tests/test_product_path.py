"""The product path (CPU only): it runs through the CUDA library or not at all.

- Without the built library every entry point raises; nothing falls back to a
  CPU implementation.
- No package source imports, loads or links the oracle (the oracle is test
  infrastructure; the library and its binding share nothing with it)."""
import os
import re

import pytest
import torch

import nvfp4_moe_expert_topk_b200 as pkg

PKG_DIR = os.path.dirname(os.path.abspath(pkg.__file__))


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(pkg, "LIB_PATH", str(tmp_path / "libnvfp4moe.so"))
    monkeypatch.setattr(pkg, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        pkg.nvfp4_scales_bytes(128, 256, pkg.NVFP4_SCALES_MMA)
    with pytest.raises(RuntimeError, match="missing"):
        pkg.nvfp4_moe_workspace_size(64, 6, 48, 7168, 3072)
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        pkg.nvfp4_amax(x, torch.zeros(1))


def test_host_tensors_are_rejected():
    """CPU tensors are refused before any work: there is no host code path."""
    from nvfp4_moe_expert_topk_b200 import build
    build.build()
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkg.nvfp4_amax(x, torch.zeros(1))
    logits = torch.zeros(8, 48)
    ids = torch.zeros(8, 7, dtype=torch.int32)
    w = torch.zeros(8, 7)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkg.nvfp4_moe_topk_shared(logits, 6, 1, ids, w)


def test_package_sources_do_not_use_the_oracle():
    pattern = re.compile(r"(^|\s)(import|from)\s+oracle\b|oracle\.(so|c|py)\b|[\"']oracle[/\"']|oracle_[a-z]+\(")
    checked = 0
    for dirpath, _, files in os.walk(PKG_DIR):
        for name in files:
            if not name.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                continue
            with open(os.path.join(dirpath, name)) as f:
                for i, line in enumerate(f, 1):
                    assert not pattern.search(line), f"{name}:{i}: {line.strip()}"
            checked += 1
    assert checked >= 8
