"""Host-side fault injection (RVQ_FAULT): named entry points return the given status before they
check their arguments or touch the device, so a caller's error handling can be tested without a
GPU fault.  Each case runs in a fresh process (the switch is read once)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code, fault):
    env = dict(os.environ, RVQ_FAULT=fault)
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    return out.stdout


def test_named_entry_points_return_the_injected_status():
    code = (
        "import multimodal_visual_tokenization_b200 as mvt\n"
        "b = mvt.rvq_launch_count()\n"
        "print(mvt.rvq_encode(16, 1, 8, 64, 16, 0, 16, 16, 16, 2, 16, None, 0, 16, None, None, None, 16, 1 << 20,"
        " None, 0))\n"
        "print(mvt.rvq_decode(16, 8, 2, 16, 0, 16, 64, 16, None, 0))\n"
        "print(mvt.rvq_encode_workspace_size(8, 64, 2, 16)[0])\n"
        "print(mvt.rvq_balance_sequences([3, 1, 2], 2)[0])\n"
        "print(mvt.rvq_launch_count() - b)\n")
    out = _run(code, "rvq_encode:-4,rvq_decode:-5,rvq_encode_workspace_size:-2").split()
    assert out[:3] == ["-4", "-5", "-2"]
    assert out[3] == "0"      # not named: runs normally (a host-only call)
    assert out[4] == "0"      # nothing was launched


def test_malformed_or_positive_entries_are_ignored():
    code = ("import multimodal_visual_tokenization_b200 as mvt\n"
            "print(mvt.rvq_balance_sequences([3, 1, 2], 2)[0])\n")
    assert _run(code, "rvq_balance_sequences:5,garbage,rvq_balance_sequences").split() == ["0"]
    assert _run(code, "rvq_balance_sequences:-3").split() == ["-3"]


@pytest.mark.gpu
def test_tokenizer_raises_the_injected_status_and_other_calls_still_work():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    code = (
        "import torch, workloads\n"
        "import multimodal_visual_tokenization_b200 as mvt\n"
        "g = workloads.generate('tiny')\n"
        "tok = mvt.Tokenizer(torch.from_numpy(g['codebooks']).cuda())\n"
        "x = torch.from_numpy(g['x']).cuda()\n"
        "try:\n"
        "    tok.encode(x)\n"
        "    print('no error')\n"
        "except mvt.RVQError as e:\n"
        "    print('raised', e.code)\n"
        "ids = torch.from_numpy(g['planted']).cuda()\n"
        "rec = tok.decode(ids)\n"
        "torch.cuda.synchronize()\n"
        "print('decode ok', rec.shape[0])\n")
    out = _run(code, "rvq_encode:-6")
    assert "raised -6" in out and "decode ok 256" in out
