"""Static checks of the launch-chaining discipline in the CUDA sources (CPU).

Kernels of one Lloyd iteration are launched with programmatic stream
serialization, which is only safe when (1) every such kernel waits on the
device (griddepcontrol.wait, `pdl_wait()`) before it can return or touch data
an earlier kernel wrote, and (2) no kernel chains to anything but another of
these kernels: every memset, copy, event or stream wait issued by the ABI
layer, and every plain `<<<>>>` launcher, breaks the chain first.  A one-
iteration fit whose first assignment chained behind the memset that clears
the sort counts returned wrong centroids on the GPU; these checks keep that
class of mistake from coming back unnoticed.
"""

import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "means_clustering_flashassign_b200", "csrc")

# Kernels launched through launch_chained (or, for the assignment, with the
# programmatic attribute set by hand).
CHAINED = ["k_assign", "k_sort_count", "k_sort_colscan", "k_sort_scatter", "k_bounds", "k_segsum",
           "k_finalize", "k_small_update"]


def _src(name):
    with open(os.path.join(CSRC, name)) as f:
        text = f.read()
    return re.sub(r"//[^\n]*", "", text)  # drop line comments (they may hold braces)


def _all_sources():
    return {n: _src(n) for n in sorted(os.listdir(CSRC)) if n.endswith((".cu", ".cuh", ".h"))}


def _body(text, start):
    """The brace-balanced body that starts at the first '{' after `start`."""
    i = text.index("{", start)
    depth = 0
    for j in range(i, len(text)):
        if text[j] == "{":
            depth += 1
        elif text[j] == "}":
            depth -= 1
            if depth == 0:
                return text[i + 1:j]
    raise AssertionError("unbalanced braces")


def _kernel_bodies(name):
    out = []
    for fname, text in _all_sources().items():
        for m in re.finditer(r"__global__[^;{]*?\b" + name + r"\s*\(", text):
            out.append((fname, _body(text, m.end())))
    return out


@pytest.mark.parametrize("kernel", CHAINED)
def test_chained_kernels_wait_before_they_can_return(kernel):
    bodies = _kernel_bodies(kernel)
    assert bodies, f"{kernel} not found"
    for fname, body in bodies:
        w = body.find("pdl_wait();")
        assert w >= 0, f"{kernel} ({fname}) never waits on the device"
        assert "return" not in body[:w], f"{kernel} ({fname}) may return before pdl_wait()"


def test_assignment_kernel_does_not_release_dependents_early():
    # measured: signalling launch_dependents at the assignment's start made the
    # iteration 14 us slower at N=1M, K=1024
    for fname, body in _kernel_bodies("k_assign"):
        assert "pdl_trigger" not in body, fname


def test_abi_layer_breaks_the_chain_after_every_stream_operation():
    text = _src("km_api.cu")
    ops = list(re.finditer(r"\b(cudaMemsetAsync|cudaMemcpyAsync|cudaEventRecord|cudaEventRecordWithFlags|cudaStreamWaitEvent)\(", text))
    assert len(ops) >= 10
    for m in ops:
        end = text.index(";", m.end())  # end of the statement holding the call
        nxt = text[end + 1:].lstrip()
        assert nxt.startswith("chain_break();"), text[m.start():end + 40]


def test_abi_entry_preparation_breaks_the_chain():
    text = _src("km_api.cu")
    m = re.search(r"\bint prepare\s*\(", text)
    assert m, "prepare() not found"
    assert "chain_break();" in _body(text, m.end())


def test_plain_launchers_break_the_chain_first():
    # every function holding a plain <<<>>> launch is a launcher that breaks
    # the chain on entry, or a helper called only from such a launcher
    for fname, text in _all_sources().items():
        if "<<<" not in text:
            continue
        heads = list(re.finditer(r"\n(?:static\s+)?(?:cudaError_t|int|void)\s+(\w+)\s*\([^;{]*\)\s*\{", text))
        for h in heads:
            body = _body(text, h.end() - 1)
            if "<<<" not in body:
                continue
            name = h.group(1)
            if body.lstrip().startswith("chain_break();"):
                continue
            callers = [g for g in heads if g is not h and re.search(r"\b" + name + r"\s*[<(]",
                                                                    _body(text, g.end() - 1))]
            assert callers, f"{fname}: {name} launches plainly and is neither a breaking launcher nor a helper"
            for g in callers:
                assert _body(text, g.end() - 1).lstrip().startswith("chain_break();"), \
                    f"{fname}: {name} is called from {g.group(1)}, which does not break the chain first"


def test_chained_launch_helper_arms_and_breaks():
    text = _src("km_internal.h")
    m = re.search(r"launch_chained\s*\(", text)
    body = _body(text, m.end())
    assert "chain_armed()" in body and "chain_arm();" in body and "chain_break();" in body


def test_scatter_reads_the_arrays_both_sort_passes_rewrite_through_l2():
    # The rank buffer and the digit totals are read by the first pass's
    # scatter and rewritten by the second pass before its scatter reads them;
    # chained kernels become resident early, so those reads must bypass the
    # non-coherent L1 path (a stale first-pass line broke repeated two-pass
    # fits' bit-identity on the GPU).
    text = _src("k_sort.cu")
    start = text.index("k_sort_scatter(")
    body = _body(text, start)
    # the ranks (both passes) through L2; the plain key read is the
    # unranked first pass's, whose keys (the assignment) no kernel of the
    # iteration rewrites
    assert body.count("__ldcg(keys_in + i)") == 2
    assert re.search(r"ld_run_l2<RPT>\(segtot", body)
    assert re.search(r"ld_run_l2<RPT>\(boff", body)
    assert not re.search(r"ld_run<RPT>\(segtot", body)
