"""The bench's staleness check for committed ncu captures: sources hashed without their
comments, so a comment edit keeps a capture, a code edit does not."""
import bench


def test_strip_comments_keeps_code_and_literals():
    src = 'int a = 1; // note\n/* block\n */ const char *u = "http://x/*y*/"; char c = \'/\';\n'
    out = bench.strip_comments(src)
    assert "note" not in out and "block" not in out
    assert '"http://x/*y*/"' in out and "'/'" in out and "int a = 1;" in out


def test_comment_edits_do_not_change_the_stripped_text_but_code_edits_do():
    a = "int f(int x) { return x + 1; } // adds one\n"
    b = "int f(int x) { return x + 1; } // increments\n"
    c = "int f(int x) { return x + 2; } // adds one\n"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)


def test_every_capture_names_a_kernel_family():
    import json, os
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")))
    for kernel, entries in rec.items():
        if kernel.startswith("_"):
            continue
        assert bench.kernel_sources(kernel)
        for e in entries:
            assert {"source_sha", "T", "B", "H", "D", "dtype", "dram_bytes_per_launch"} <= set(e)


def test_causal_workload_keeps_its_unit_decay_through_resizing():
    import synth
    w = synth.WORKLOADS["causal_bf16"].with_T(130)
    inp = synth.make_inputs(w, seed=1)
    assert w.extra == {"gamma": 1.0}
    assert inp["gamma"].tolist() == [1.0] * w.H
    assert tuple(inp["q"].shape) == (w.B, w.H, 130, 64)
