"""The library's debug knobs (no GPU needed): AWQ_LOG=1 traces every
device-side call and every non-OK status on stderr; AWQ_FAULT injects a host
fault at a call's entry (bad argument, short workspace, failed launch) before
any check or launch.  Each case runs in a fresh interpreter, since the
library reads both variables once."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# A fake device address (16-byte aligned) the calls never dereference.
SCRIPT = r'''
import ctypes, sys
sys.path.insert(0, {root!r})
from post_weight_only_b200 import build
lib = ctypes.CDLL(build.build())
P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
fake = 1 << 40
lib.awq_get_last_error.restype = ctypes.c_char_p
lib.awq_act_stats.argtypes = [P, I64, I64, I, P, P]
lib.awq_quantize_pack.argtypes = [P, P, I64, I64, I, I, P, P, P]
lib.awq_search.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, I, P, P, P, P, P, SZ, P, P]
lib.awq_search.restype = I
rc = {{}}
rc["act_stats_null"] = lib.awq_act_stats(None, 16, 64, 0, fake, None)
rc["act_stats"] = lib.awq_act_stats(fake, 16, 64, 0, fake, None)
rc["pack"] = lib.awq_quantize_pack(fake, fake, 256, 64, 4, 128, fake, fake, None)
rc["search"] = lib.awq_search(fake, fake, fake, 16, 256, 64, fake, 3, 4, 128, 0, fake, None, fake, fake,
                              fake, 1 << 30, fake, None)
rc["msg"] = lib.awq_get_last_error().decode()
print(repr(rc))
'''


def run(env_extra):
    env = dict(os.environ)
    env.pop("AWQ_LOG", None)
    env.pop("AWQ_FAULT", None)
    env.update(env_extra)
    env["CUDA_VISIBLE_DEVICES"] = ""            # host paths only, on any machine
    out = subprocess.run([sys.executable, "-c", SCRIPT.format(root=ROOT)], env=env, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr
    return eval(out.stdout.strip().splitlines()[-1]), out.stderr


def test_log_traces_calls_and_failures():
    rc, err = run({"AWQ_LOG": "1"})
    assert rc["act_stats_null"] == 1                          # NULL X: AWQ_EINVAL, as without the knob
    assert "[awq] awq_act_stats(N=16 D_in=64 stat=0)" in err
    assert "[awq]   -> status 1:" in err
    assert "[awq] awq_quantize_pack(D_in=256 D_out=64 bits=4 group=128)" in err
    assert "[awq] awq_search(N=16 D_in=256 D_out=64 n_alpha=3 bits=4 group=128 form=0)" in err


def test_no_trace_without_the_knob():
    _, err = run({})
    assert "[awq]" not in err


@pytest.mark.parametrize("mode,code,who", [("badarg", 1, "pack"), ("workspace", 4, "search"), ("alloc", 4, "search"),
                                           ("launch", 5, "act_stats")])
def test_fault_injection(mode, code, who):
    rc, _ = run({"AWQ_FAULT": mode})
    assert rc[who] == code
    assert f"AWQ_FAULT={'workspace' if mode == 'alloc' else mode} (injected)" in rc["msg"] or mode == "launch"


def test_workspace_fault_spares_calls_without_a_workspace():
    rc, _ = run({"AWQ_FAULT": "workspace"})
    assert rc["act_stats_null"] == 1                          # its own argument check, not the injected fault
    assert rc["pack"] != 4


def test_launch_fault_names_the_launch_failure():
    rc, _ = run({"AWQ_FAULT": "launch"})
    assert rc["search"] == 5
    assert "AWQ_FAULT=launch (injected): cudaErrorLaunchFailure" in rc["msg"]
