"""Source rules the kernels keep, checked on the text of csrc/ (no GPU).

Every kernel is launched as a programmatic dependent of the one before it and triggers
its dependents first. A kernel can therefore be resident while its predecessors still
write its inputs. Loads through `const __restrict__` pointers or `__ldg` compile to the
non-coherent form, which is only valid for memory that no one writes while the kernel
lives. So those qualifiers may mark only weights. The caller's x may itself be the output
of this library's previous call on the stream (two layers stacked back to back), so it is
read with plain loads like every other activation."""
import pathlib
import re

CSRC = pathlib.Path(__file__).resolve().parents[1] / "mixture_experts_layer_29_b200" / "csrc"

# weights: no kernel of this library writes them
READ_ONLY_NAMES = {"w", "wgu", "wd"}
# k_split_router_weight writes a bf16 copy of the router weight through `out`
WRITE_ONLY = {("gemm_tc.cu", "out")}


def _sources():
    files = sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh"))
    assert files
    return [(f.name, f.read_text()) for f in files]


def test_restrict_marks_only_inputs_and_weights():
    bad = []
    for name, text in _sources():
        for m in re.finditer(r"__restrict__\s+(\w+)", text):
            p = m.group(1)
            if p not in READ_ONLY_NAMES and (name, p) not in WRITE_ONLY:
                line = text.count("\n", 0, m.start()) + 1
                bad.append(f"{name}:{line} {p}")
    assert not bad, bad


def test_no_ldg():
    for name, text in _sources():
        assert "__ldg(" not in text, name


def test_no_environment_reads():
    """Kernel choices come from the call's arguments and moe_set_tuning, never from the
    process environment."""
    for name, text in _sources():
        assert "getenv" not in text, name
