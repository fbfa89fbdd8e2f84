"""The leaf-structure autotune cache (JSON keyed by m, n, bits, GPU name):
host logic only."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import two_sided_gptq_b200 as bk  # noqa: E402


def test_round_trip_and_keys(tmp_path):
    path = str(tmp_path / "tune.json")
    k1 = bk.tune_cache_key(4096, 4096, 4, "NVIDIA B200")
    k2 = bk.tune_cache_key(4096, 4096, 3, "NVIDIA B200")
    assert k1 != k2 and k1 != bk.tune_cache_key(4096, 4096, 4, "other GPU")
    assert bk.tune_cache_get(path, k1) is None  # no file yet
    bk.tune_cache_put(path, k1, 3, [17.0, 19.6, 8.7, 9.4])
    bk.tune_cache_put(path, k2, 4, [1, 2, 3, 0.5])
    assert bk.tune_cache_get(path, k1) == (3, [17.0, 19.6, 8.7, 9.4])
    assert bk.tune_cache_get(path, k2) == (4, [1.0, 2.0, 3.0, 0.5])
    assert set(json.load(open(path))) == {k1, k2}
    assert not [f for f in os.listdir(tmp_path) if f.startswith(".bakron_tune_")]  # no temporary left


def test_bad_files_and_entries_are_misses(tmp_path):
    path = str(tmp_path / "tune.json")
    open(path, "w").write("{not json")
    assert bk.tune_cache_get(path, "k") is None
    bk.tune_cache_put(path, "k", 2, [1.0])  # a corrupt file is replaced
    assert bk.tune_cache_get(path, "k") == (2, [1.0])
    json.dump({"k": {"leaf": 9, "ms": []}, "j": "x"}, open(path, "w"))  # no structure 9
    assert bk.tune_cache_get(path, "k") is None and bk.tune_cache_get(path, "j") is None
