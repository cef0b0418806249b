"""Host-side logic of bench.py (no GPU): the L2-cold replica count, the step
count, and the lookup of the committed ncu traffic figure by source hash."""
from __future__ import annotations

import hashlib
import os

import bench
from bit_recurrent_state_decode_b200 import synth


def test_replicas_exceed_four_l2():
    l2 = 126_000_000
    for name, wl in synth.WORKLOADS.items():
        per_layer = 20_000_000
        r = bench.pick_replicas(wl, l2, per_layer)
        if wl.layers > 1:
            assert r == 1, name            # already many layers: stepped as stated
        else:
            assert r * per_layer >= 4 * l2 and (r - 1) * per_layer < 4 * l2, name


def test_default_steps():
    assert bench.default_steps(1.0) == 50          # never fewer than 50
    assert 29_990 <= bench.default_steps(1e-4) <= 30_000   # about 3 s of timed work
    assert bench.default_steps(0.0) > 0


def _fake_root(tmp_path, profile_hash, value="123456"):
    csrc = tmp_path / "bit_recurrent_state_decode_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cuh").write_bytes(b"kernel source A")
    (csrc / "b.cu").write_bytes(b"kernel source B")
    (csrc / "notes.txt").write_bytes(b"not hashed")
    digest = bench.source_digest(str(csrc))
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "step_kernel_w.md").write_text(
        f"# summary\n\n- source_sha256_16: `{profile_hash or digest}`\n"
        f"- dram_bytes_per_launch_full_size: {value}\n"
        f"- tiles_per_launch_full_size: 1000\n")
    return digest


def test_traffic_read_when_sources_match(tmp_path, monkeypatch):
    _fake_root(tmp_path, None)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_traffic("w") == 123456.0
    assert bench.read_traffic("missing") is None


def test_traffic_scaled_to_the_launch_by_tiles(tmp_path, monkeypatch):
    """A launch of another size (other --layers / --replicas) gets the
    committed full-size traffic scaled by its tile count, not the full-size
    figure itself."""
    _fake_root(tmp_path, None)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_traffic("w", 1000) == 123456.0
    assert bench.read_traffic("w", 250) == 123456.0 / 4


def test_traffic_null_once_the_kernel_changes(tmp_path, monkeypatch):
    _fake_root(tmp_path, "0000000000000000")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_traffic("w") is None


def test_committed_profiles_name_their_kernel_and_command():
    prof = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles")
    files = [f for f in os.listdir(prof) if f.endswith(".md")]
    assert files
    for f in files:
        text = open(os.path.join(prof, f)).read()
        if f.startswith("ptxas_"):
            # the compiler's resource report: its command, on committed units
            assert "nvcc " in text and "-Xptxas -v" in text and "bit_recurrent_state_decode_b200/csrc/" in text
            continue
        assert f.split("_kernel_")[0] in ("step", "rows", "lrb", "pw", "rc"), f
        assert "source_sha256_16:" in text and "dram_bytes_per_launch_full_size:" in text
        assert "ncu " in text and "--clock-control none" in text and "python bench.py" in text


def test_source_digest_is_of_the_code(tmp_path):
    """Comments and whitespace do not change the digest that ties a profile
    to the kernel sources; code, a file name, or a // inside a string
    literal does."""
    d = tmp_path / "csrc"
    d.mkdir()
    f = d / "k.cuh"

    def digest(text, name="k.cuh"):
        for p in d.iterdir():
            p.unlink()
        (d / name).write_text(text)
        return bench.source_digest(str(d))

    base = digest('int x = 1;  // the count\nconst char* s = "a//b"; /* it\'s */ char c = \'/\';\n')
    assert digest('int x = 1;\n\n   const char* s = "a//b";\nchar c = \'/\'; // other words\n') == base
    assert digest('int x = 2; const char* s = "a//b"; char c = \'/\';') != base
    assert digest('int x = 1; const char* s = "a/ /b"; char c = \'/\';') != base
    assert digest('int x = 1; const char* s = "a//b"; char c = \'/\';', name="j.cuh") != base
    assert digest('int x = 1; const char* s = "a//b"; char c = \'/\';') == base
    (d / "notes.txt").write_text("not a source")
    assert bench.source_digest(str(d)) == base
