"""The debug library (libmsa_debug.so) on a GPU, in a child process that loads
it alone (MSA_DEBUG=1): a valid fp32 chain runs clean; non-decreasing
offsets that go backwards, and a memory length above m_cap, are refused by
the call that receives them (MSA_ERR_INVALID_ARG) before any kernel reads
through them; a gather that overflows its capacity returns MSA_ERR_CAPACITY
from the call itself.

Nothing here can fault the GPU: every bad array is refused by the call's
device-side check before a kernel reads through it, and the overflowing
gather caps its writes at m_cap.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import torch
from latent_memory_routing_b200 import msa, pipeline, synth

assert msa.LIB_PATH.endswith("libmsa_debug.so"), msa.LIB_PATH
msa.lib()
msa.msa_device_status(clear=True)

def refused(fn, code):
    try:
        fn()
    except msa.MsaError as e:
        assert e.status == code, (e.status, code)
        assert msa.msa_device_status(clear=True) in (0, code)
        return
    raise AssertionError("the call was not refused")

# a valid fp32 chain: encode -> route -> top-k -> gather -> attend
w = synth.tiny("cuda")
toff = w["tok_offsets"].cuda()
coff = pipeline.chunk_offsets(toff)
kb, vb, rb = pipeline.encode_pool(w["k_tok"], w["v_tok"], w["kr_tok"], toff, coff, 48)
p = pipeline.Pipeline(rb[0], kb[0], vb[0], coff, B=1, T=16, T_loc=16, Hq=4, k=2, m_cap=6)
out = p(w["q_r"], w["q"], w["k_loc"], w["v_loc"])
torch.cuda.synchronize()
assert bool(torch.isfinite(out).all())
assert msa.msa_device_status(clear=True) == 0

# offsets that go backwards: refused by the pooling call itself
bad = toff.clone()
bad[3] = bad[5]
refused(lambda: pipeline.encode_pool(w["k_tok"], w["v_tok"], w["kr_tok"], bad, coff, 48), -1)

# a memory length above m_cap: refused by the attention call
ml = torch.tensor([7], dtype=torch.int32, device="cuda")
att = pipeline.Attention(torch.float32, 1, 16, 16, 4, 2, 64, 6, "cuda")
refused(lambda: att(w["q"], p.k_mem, p.v_mem, ml, w["k_loc"], w["v_loc"], 2), -1)

# a gather past its capacity: MSA_ERR_CAPACITY from the call
idx = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
refused(lambda: pipeline.gather_kv(idx, coff, kb[0], vb[0], 4), -3)

# and the library keeps working afterwards
out2 = p(w["q_r"], w["q"], w["k_loc"], w["v_loc"])
torch.cuda.synchronize()
assert torch.equal(out, out2)
assert msa.msa_device_status(clear=True) == 0
print("debug build ok")
"""


def test_debug_library_refuses_bad_index_arrays(cuda_device):
    from latent_memory_routing_b200 import build
    build.build(debug=True)
    env = dict(os.environ, MSA_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout
