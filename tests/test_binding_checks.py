"""The binding's marshalling checks (no GPU needed): a tensor the C ABI
cannot take as a plain device pointer -- wrong dtype, rank, size or layout,
or memory the kernels cannot dereference -- is rejected in Python before
any library call."""
import numpy as np
import pytest

import ternary_moe_butterfly_b200 as bf

torch = pytest.importorskip("torch")

d, N, k, T = 64, 4, 2, 8
L = 6


def args(**over):
    a = dict(
        x=torch.zeros((T, d), dtype=torch.float32),
        logits=torch.zeros((T, N), dtype=torch.float32),
        packed=torch.zeros(bf.bfmoe_packed_base_bytes(d), dtype=torch.uint8),
        theta=torch.zeros((N, L, d // 2), dtype=torch.float32),
        phi=torch.zeros((N, L, d // 2), dtype=torch.float32),
    )
    a.update(over)
    return a


def call_forward(**over):
    a = args(**over)
    return bf.forward(a["x"], a["logits"], k, a["packed"], a["theta"], a["phi"], ws=a.get("ws"), out=a.get("out"))


def test_forward_rejects_host_memory():
    with pytest.raises(ValueError, match="CUDA"):
        call_forward()


@pytest.mark.parametrize("over,exc,msg", [
    (dict(logits=torch.zeros((T, N), dtype=torch.float64)), TypeError, "logits"),
    (dict(x=torch.zeros((T, d), dtype=torch.float16)), TypeError, "float32 or bfloat16"),
    (dict(x=torch.zeros((d, T), dtype=torch.float32).t()), ValueError, "contiguous"),
    (dict(x=torch.zeros(T * d, dtype=torch.float32)), ValueError, "dimensions"),
    (dict(logits=torch.zeros((T + 1, N), dtype=torch.float32)), ValueError, "rows"),
    (dict(theta=torch.zeros((N, L - 1, d // 2), dtype=torch.float32)), ValueError, "theta"),
    (dict(phi=torch.zeros((N, L, d // 2), dtype=torch.float64)), TypeError, "phi"),
    (dict(packed=torch.zeros(16, dtype=torch.uint8)), ValueError, "packed"),
    (dict(out=torch.zeros((T, d), dtype=torch.bfloat16)), TypeError, "out"),
    (dict(ws=torch.zeros(1024, dtype=torch.int32)), TypeError, "ws"),
    (dict(theta=np.zeros((N, L, d // 2), np.float32)), TypeError, "theta"),
])
def test_forward_rejects_bad_tensors(over, exc, msg):
    with pytest.raises(exc, match=msg):
        call_forward(**over)


def test_butterfly_apply_checks():
    x = torch.zeros((5, d), dtype=torch.float32)
    ang = torch.zeros((N, L, d // 2), dtype=torch.float32)
    with pytest.raises(TypeError, match="expert_of_row"):
        bf.butterfly_apply(x, ang, torch.zeros(5, dtype=torch.int64))
    with pytest.raises(ValueError, match="expert_of_row"):
        bf.butterfly_apply(x, ang, torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError, match="angles"):
        bf.butterfly_apply(x, torch.zeros((N, L, d), dtype=torch.float32))
    with pytest.raises(ValueError, match="CUDA"):
        bf.butterfly_apply(x, ang, torch.zeros(5, dtype=torch.int32))


def test_route_and_pack_checks():
    with pytest.raises(ValueError, match="dimensions"):
        bf.route(torch.zeros(T * N, dtype=torch.float32), k)
    with pytest.raises(TypeError, match="logits"):
        bf.route(torch.zeros((T, N), dtype=torch.float16), k)
    with pytest.raises(ValueError, match="CUDA"):
        bf.route(torch.zeros((T, N), dtype=torch.float32), k)
    with pytest.raises(TypeError, match="int8"):
        bf.pack_base(torch.zeros((d, d), dtype=torch.int32), 1.0)
    with pytest.raises(ValueError, match="square"):
        bf.pack_base(torch.zeros((d, d + 1), dtype=torch.int8), 1.0)
    with pytest.raises(ValueError, match="CUDA"):
        bf.pack_base(torch.zeros((d, d), dtype=torch.int8), 1.0)
