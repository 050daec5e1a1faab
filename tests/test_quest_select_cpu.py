"""The page-level comparator's selection (quest_select in
query_aware_kv_ts_b200/csrc/quest.cu, one 8-CTA cluster per sequence) on the
CPU: the kernel's own source, its constants and the order key it uses,
compiled for the host by tests/quest_select_emu.cpp (every __shared__
declaration given per-CTA storage, the cluster's shared memory mapped
between CTAs) and run on seeded page scores; the rows and counts must equal
the oracle's quest_select exactly.  The cases reach both of the kernel's
paths: the fast one (at most 2048 chosen pages, at most 2048 pages in the
threshold's bin) and the general one (more tied pages, or more chosen pages,
than that), with ragged and empty sequences, one-token pages, ties between
+0 and -0 and integer-valued scores.  A guard on the selection's logic that
needs no GPU (the GPU tests run the same kernel on the device)."""
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "query_aware_kv_ts_b200", "csrc")
HARNESS = os.path.join(ROOT, "tests", "quest_select_emu.cpp")


def _function(src: str, signature: str) -> str:
    """From `signature` to the function's closing brace (a line of its own)."""
    a = src.index(signature)
    return src[a:src.index("\n}\n", a) + 3]


def kernel_sources():
    """(order key, constants, selection source with per-CTA shared storage)."""
    with open(os.path.join(CSRC, "score_common.cuh")) as f:
        order_key = _function(f.read(), "__device__ __forceinline__ int32_t float_order_key")
    with open(os.path.join(CSRC, "quest.cu")) as f:
        src = f.read()
    constants = "\n".join(re.findall(r"^constexpr int kQuestSel\w+ = [^;]+;", src, re.M)) + "\n"
    start = src.index("// Exclusive prefix sum of one value per thread over the CTA")
    sig = src.index("quest_select(const float *scores")
    body = src[start:src.index("\n}\n", sig) + 3]
    decl = [0]

    def per_cta(m):
        typ, names = m.group(1), m.group(2)
        out = []
        for name in (x.strip() for x in names.split(",")):
            decl[0] += 1
            arr = re.match(r"(\w+)\[(.+)\]$", name)
            if arr:
                out.append("%s *%s = emu_shared<%s>(%d, (size_t)(%s));" % (typ, arr.group(1), typ, decl[0],
                                                                          arr.group(2)))
            else:
                out.append("%s &%s = *emu_shared<%s>(%d, 1);" % (typ, name, typ, decl[0]))
        return " ".join(out)

    body = re.sub(r"__shared__\s+([\w:]+)\s+([^;]+);", per_cta, body)
    return order_key, constants, body, decl[0]


def test_kernel_sources_are_found():
    order_key, constants, body, decls = kernel_sources()
    assert "float_order_key" in order_key and "kQuestSelThreads" in constants and "kQuestSelBins" in constants
    assert "__shared__" not in body and decls > 0 and body.rstrip().endswith("}")


def _cases():
    """(name, lengths, log2 P, k, n_sink, n_local, scores drawn by rng)."""
    return [
        ("ragged_p16", [5000, 777], 4, 512, 4, 128, lambda r, n: r.standard_normal(n)),
        ("empty_and_tiny_p16", [0, 500, 0, 1], 4, 32, 4, 8, lambda r, n: r.standard_normal(n)),
        ("one_token_pages", [700], 0, 64, 4, 16, lambda r, n: r.standard_normal(n)),
        ("integer_scores_p8", [2000], 3, 200, 4, 64, lambda r, n: r.integers(-3, 4, n).astype(float)),
        ("signed_zeros", [1600], 2, 120, 4, 32, lambda r, n: np.where(r.integers(0, 2, n) == 1, 0.0, -0.0)),
        # the general path: more than 2048 pages tied in the threshold's bin,
        # and more than 2048 pages to choose
        ("general_all_tied", [5000], 0, 100, 4, 16, lambda r, n: np.full(n, 1.5)),
        ("general_large_budget", [8000, 300], 0, 3000, 4, 64, lambda r, n: r.standard_normal(n)),
    ]


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_selection_matches_the_oracle(tmp_path):
    order_key, constants, body, _ = kernel_sources()
    (tmp_path / "order_key.inc").write_text(order_key)
    (tmp_path / "constants.inc").write_text(constants)
    (tmp_path / "select.inc").write_text(body)
    exe = str(tmp_path / "quest_select_emu")
    subprocess.run(["g++", "-std=c++20", "-O1", "-pthread", "-I", str(tmp_path), HARNESS, "-o", exe], check=True,
                   capture_output=True, timeout=300)
    for i, (name, lengths, p_shift, k, s, l, draw) in enumerate(_cases()):
        P = 1 << p_shift
        off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
        B = len(lengths)
        rows = int((off[-1] // P + B + 3) // 4 * 4)
        scores = np.asarray(draw(np.random.default_rng(100 + i), rows), np.float32)
        inp, out = tmp_path / ("%s.in" % name), tmp_path / ("%s.out" % name)
        with open(inp, "wb") as f:
            f.write(np.array([B, p_shift, k, s, l, rows], np.int64).tobytes())
            f.write(off.tobytes())
            f.write(scores.tobytes())
        run = subprocess.run([exe, str(inp), str(out)], capture_output=True, text=True, timeout=600)
        assert run.returncode == 0 and run.stdout.strip() == "ok", (name, run.stdout, run.stderr)
        cap = k + s + l
        res = np.fromfile(out, np.int32)
        ids, count = res[:B * cap].reshape(B, cap), res[B * cap:]
        for b, n in enumerate(lengths):
            r0 = int(off[b]) // P + b
            want, m = oracle.quest_select(scores[r0:r0 + oracle.quest_pages(n, P)].astype(np.float64), n, P, k, s, l)
            assert int(count[b]) == m, (name, b, count[b], m)
            assert np.array_equal(ids[b], want), (name, b)
