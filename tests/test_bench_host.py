"""Host-side helpers of bench.py: the code digest that decides whether a
recorded ncu capture still applies to the kernel (roofline.traffic), and the
records themselves."""
import json
import os

import bench

CSRC = os.path.join("ternary_weight_decoder_b200", "csrc")


def _tree_reader(overrides):
    """Reads the working tree, with some files' text replaced."""
    def read(rel):
        if rel in overrides:
            return overrides[rel]
        with open(os.path.join(bench.ROOT, rel)) as f:
            return f.read()
    return read


def test_digest_ignores_comments_and_blank_lines():
    rel = os.path.join(CSRC, "tw_decode.cu")
    text = open(os.path.join(bench.ROOT, rel)).read()
    edited = ("// a new leading comment\n\n" +
              text.replace("\n", "  \n", 5) +
              "\n/* a block\n   comment */\n")
    assert bench.code_digest("tw_decode.cu", _tree_reader({rel: edited})) == \
        bench.code_digest("tw_decode.cu")


def test_digest_sees_code_changes_in_the_kernel_and_the_headers():
    base = bench.code_digest("tw_decode.cu")
    rel = os.path.join(CSRC, "tw_decode.cu")
    text = open(os.path.join(bench.ROOT, rel)).read()
    assert "constexpr int kXE = 8;" in text
    changed = text.replace("constexpr int kXE = 8;", "constexpr int kXE = 4;")
    assert bench.code_digest("tw_decode.cu", _tree_reader({rel: changed})) != base
    hrel = os.path.join(CSRC, "tw_internal.h")
    htext = open(os.path.join(bench.ROOT, hrel)).read()
    assert bench.code_digest("tw_decode.cu", _tree_reader({hrel: htext + "\nint x;\n"})) != base


def test_strip_comments():
    src = "int a; // one\n/* two\nthree */ int b;\n\n  \nint c; /* four */\n"
    assert bench._strip_comments(src) == "int a;\n int b;\nint c;"


def test_traffic_records_are_well_formed():
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    assert d["captures"]
    for e in d["captures"]:
        assert os.path.exists(os.path.join(bench.ROOT, CSRC, e["kernel_src"]))
        assert os.path.exists(os.path.join(bench.ROOT, "profiles", e["summary"]))
        assert e["dram_bytes_per_launch"] == e["dram_read_bytes"] + e["dram_write_bytes"]
        assert len(e["code_sha256"]) == 64 and e["M"] >= 1 and e["layers"] >= 1
