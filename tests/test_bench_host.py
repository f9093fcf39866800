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


def test_kernel_sources_follow_includes_and_skip_the_public_header():
    srcs = bench.kernel_sources("tw_decode_tc.cu")
    names = [os.path.basename(s) for s in srcs]
    assert names[0] == "tw_decode_tc.cu"
    assert {"tw_device.cuh", "tw_internal.h", "tw_tc.cuh"} <= set(names)
    assert "ternary_decoder.h" not in names
    assert "tw_tc.cuh" not in [os.path.basename(s) for s in bench.kernel_sources("tw_decode.cu")]


def test_public_header_edit_keeps_the_digest():
    rel = os.path.join("include", "ternary_decoder.h")
    text = open(os.path.join(bench.ROOT, rel)).read()
    edited = text.replace("#endif /* TERNARY_DECODER_H */",
                          "int tw_new_entry(void);\n#endif /* TERNARY_DECODER_H */")
    assert edited != text
    assert bench.code_digest("tw_decode.cu", _tree_reader({rel: edited})) == \
        bench.code_digest("tw_decode.cu")


def test_dist_summary_and_cpu_info():
    s = bench.dist_summary([0.1] * 8 + [0.2, 0.3])
    assert s["median_us"] == 100.0 and s["samples"] == 10
    assert s["p10_us"] <= s["median_us"] <= s["p90_us"] <= 300.0
    info = bench.cpu_info()
    assert info["nproc"] >= 1 and info["cpus_available"] >= 1


def test_bench_arguments_default_to_one_gpu():
    a = bench.parse([])
    assert a.gpus == 1 and a.m == 1 and a.layers == 28 and a.warmup >= 3
    assert set(a.configs.split(",")) == {"1", "2", "4", "5", "mid", "i8", "chain"}
