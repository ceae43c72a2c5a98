"""The committed DRAM-traffic record is tied to the decode path's code by a
hash; these CPU tests pin what the hash sees (no GPU)."""
import json
import shutil
from pathlib import Path

import bench

CSRC = Path(bench.ROOT) / "paged_kv_cache_444_b200" / "csrc"


def _copy(tmp_path: Path) -> Path:
    dst = tmp_path / "csrc"
    shutil.copytree(CSRC, dst)
    return dst


def test_comment_edits_keep_the_hash(tmp_path):
    src = _copy(tmp_path)
    before = bench.kernel_source_digest(src)
    f = src / "pa_decode.cuh"
    text = f.read_text()
    f.write_text("// a new leading comment\n\n" +
                 text.replace("namespace pa {", "namespace pa {  // trailing comment\n/* a block\n comment */", 1))
    assert bench.kernel_source_digest(src) == before


def test_code_edits_change_the_hash(tmp_path):
    src = _copy(tmp_path)
    before = bench.kernel_source_digest(src)
    f = src / "pa_decode.cuh"
    text = f.read_text()
    assert "constexpr int kWarps = 4;" in text
    f.write_text(text.replace("constexpr int kWarps = 4;", "constexpr int kWarps = 8;", 1))
    assert bench.kernel_source_digest(src) != before


def test_files_off_the_decode_path_and_marked_regions_are_ignored(tmp_path):
    src = _copy(tmp_path)
    before = bench.kernel_source_digest(src)
    for name in bench.OFF_DECODE_PATH:
        (src / name).write_text((src / name).read_text() + "\nint changed_off_path = 1;\n")
    api = src / "pa_api.cu"
    text = api.read_text()
    marker = "\n// <<< fp8 KV cache launch"
    assert marker in text
    api.write_text(text.replace(marker, "\nint changed_inside_region = 1;" + marker, 1))
    assert bench.kernel_source_digest(src) == before


def test_the_record_matches_the_current_code():
    rec = json.loads((Path(bench.ROOT) / "profiles" / "traffic.json").read_text())
    shas = {v["source_sha"] for cfg in rec.values() if isinstance(cfg, dict)
            for v in cfg.values() if isinstance(v, dict) and "source_sha" in v}
    assert shas == {bench.kernel_source_digest()}
