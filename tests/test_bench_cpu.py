"""Host logic of bench.py (CPU only): the roofline's algorithmic bytes and the gate
that reports ncu traffic only for the kernel source it was captured from."""
import os
import shutil

import bench
import fmoe_synth as synth
import oracle


def test_layer_bytes_full_size():
    """Per token of the full-size 4-bit top-4 layer: K + 1 expert records (sizes from
    the oracle's own reading of the format), the fp32 router and shared gate vector,
    and x, the residual and y in bf16."""
    shape = synth.CONFIGS["layer4096"]["shape"]
    rec = oracle.record_regions(shape.hidden, shape.inter, shape.bits)["size"]
    experts, rest = bench.layer_bytes(shape)
    assert experts == (shape.top_k + 1) * rec == 5 * 7_077_888 == 35_389_440
    assert rest == 512 * 4096 * 4 + 4096 * 4 + 3 * 4096 * 2 == 8_429_568
    assert experts + rest == 43_819_008


def test_layer_bytes_two_bit_and_no_shared():
    shape = synth.LayerShape(4096, 1024, 512, 4, 2, 0, 0)
    experts, rest = bench.layer_bytes(shape)
    assert experts == 4 * oracle.record_regions(4096, 1024, 2)["size"] == 4 * 3_932_160
    assert rest == 512 * 4096 * 4 + 3 * 4096 * 2


def test_kernel_source_digest_ignores_comments_and_spacing():
    a = bench.kernel_source_digest(["int a = 1; // first\n/* block\ncomment */ int b;"])
    b = bench.kernel_source_digest(["int  a = 1;   // changed\n int b;"])
    c = bench.kernel_source_digest(["int a = 2; int b;"])
    assert a == b and a != c
    # file boundaries and order count
    assert bench.kernel_source_digest(["int a;", "int b;"]) != bench.kernel_source_digest(["int b;", "int a;"])


def test_profiled_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    root = tmp_path
    csrc = root / "bit_dequant_expert_softmax_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    src_dir = os.path.join(bench.ROOT, "bit_dequant_expert_softmax_b200", "csrc")
    for f in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(src_dir, f), csrc / f)
    texts = [(csrc / f).read_text() for f in bench.KERNEL_SOURCES]
    (root / "profiles" / "fmoe_layer_kernel_layer4096.md").write_text(
        "summary\n\n    kernel_source_digest: %s\n    traffic_bytes_per_launch: 123456\n"
        % bench.kernel_source_digest(texts))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.profiled_traffic() == 123456
    first = csrc / bench.KERNEL_SOURCES[0]
    first.write_text(first.read_text() + "\n// a comment only\n")
    assert bench.profiled_traffic() == 123456
    first.write_text(first.read_text() + "\nnamespace fmoe { constexpr int kChanged = 1; }\n")
    assert bench.profiled_traffic() is None


def test_committed_profiles_match_the_kernel_sources():
    """The ncu summaries the bench line takes its DRAM traffic from were captured from
    the kernel sources as they are (a kernel change needs a new capture)."""
    import bench
    assert bench.profiled_traffic() is not None
    assert bench.profiled_traffic("traffic_warm_bytes_per_launch") is not None
    assert bench.profiled_traffic(summary="gdn_step_kernel_gdn45.md", sources=("fmoe_gdn.cuh",)) is not None
