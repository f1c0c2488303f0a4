"""Source rules of the CUDA kernels that no compiler flag enforces (CPU only).

A persistent kernel reads, after an acquire on an event, data that other SMs wrote during
the same launch.  Such a load must stay after the acquire in program order.  The __ldcg
intrinsics are plain inline asm without a memory clobber, so the compiler is free to
schedule them before the acquire; the kernels use the ordered ldcg_* loads instead."""
import pathlib
import re

CSRC = pathlib.Path(__file__).resolve().parents[1] / "persistent_megakernel_decode_04_b200" / "csrc"


def _sources():
    return sorted(list(CSRC.glob("*.cu")) + list(CSRC.glob("*.cuh")))


def test_no_unordered_coherent_loads():
    bad = []
    for p in _sources():
        for n, line in enumerate(p.read_text().splitlines(), 1):
            if re.search(r"\b__ld(cg|cv|cs|lu)\s*\(", line):
                bad.append(f"{p.name}:{n}: {line.strip()}")
    assert not bad, "use the ordered ldcg_* loads:\n" + "\n".join(bad)


def test_ordered_loads_are_volatile_with_a_memory_clobber():
    text = (CSRC / "mk_ptx.cuh").read_text()
    bodies = re.findall(r"ldcg_\w+\([^)]*\)\s*\{(.*?)\n\}", text, flags=re.S)
    assert len(bodies) >= 5
    for b in bodies:
        assert "asm volatile" in b and '"memory"' in b, b
