"""Pins of the gen-tower SwiGLU MLP oracle against facts outside it: torch's
own silu and linear layers, torch autograd, finite differences and closed-form
special cases. CPU only."""
import numpy as np
import pytest
import torch

from oracle import mot_mlp_oracle as M

pytestmark = pytest.mark.filterwarnings("ignore")


def _weights(rng, d, inter, r, lora=True):
    w = {
        "w_gate": rng.normal(0, 0.3, (inter, d)),
        "w_up": rng.normal(0, 0.3, (inter, d)),
        "w_down": rng.normal(0, 0.3, (d, inter)),
    }
    if lora:
        w.update({
            "a_gate": rng.normal(0, 0.5, (r, d)), "b_gate": rng.normal(0, 0.5, (inter, r)),
            "a_up": rng.normal(0, 0.5, (r, d)), "b_up": rng.normal(0, 0.5, (inter, r)),
            "a_down": rng.normal(0, 0.5, (r, inter)), "b_down": rng.normal(0, 0.5, (d, r)),
        })
    return w


def _torch_mlp(x, w, s, lora=True):
    """The block composed from torch library routines (F.linear, F.silu)."""
    F = torch.nn.functional
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=k.startswith(("a_", "b_"))) for k, v in w.items()}
    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)

    def lin(inp, name):
        y = F.linear(inp, t["w_" + name])
        if lora:
            y = y + s * F.linear(F.linear(inp, t["a_" + name]), t["b_" + name])
        return y

    g = lin(xt, "gate")
    u = lin(xt, "up")
    y = lin(F.silu(g) * u, "down")
    return xt, t, y


def test_silu_matches_torch_and_closed_forms():
    z = np.concatenate([np.linspace(-40, 40, 2001), [0.0, 1e-8, -1e-8, 700.0, -700.0]])
    ref = torch.nn.functional.silu(torch.tensor(z, dtype=torch.float64)).numpy()
    np.testing.assert_allclose(M.silu(z), ref, rtol=1e-14, atol=1e-300)
    assert M.silu(0.0) == 0.0
    assert M.silu(700.0) == 700.0  # sigmoid -> 1
    assert abs(M.silu(-700.0)) < 1e-290  # sigmoid -> 0 without overflow
    # silu(z) - silu(-z) = z (since sigmoid(z) + sigmoid(-z) = 1)
    np.testing.assert_allclose(M.silu(z) - M.silu(-z), z, rtol=1e-12, atol=1e-12)


def test_silu_grad_matches_finite_differences():
    z = np.linspace(-12, 12, 481)
    h = 1e-6
    fd = (M.silu(z + h) - M.silu(z - h)) / (2 * h)
    np.testing.assert_allclose(M.silu_grad(z), fd, rtol=1e-7, atol=1e-9)
    assert M.silu_grad(0.0) == 0.5


@pytest.mark.parametrize("lora", [True, False])
def test_forward_matches_torch_composition(lora):
    rng = np.random.default_rng(3)
    d, inter, r, s = 12, 20, 3, 0.7
    w = _weights(rng, d, inter, r, lora)
    x = rng.normal(0, 1, (2, 5, d))
    got = M.mlp_forward(x, w, s)
    _, _, y = _torch_mlp(x, w, s, lora)
    np.testing.assert_allclose(got["y"], y.detach().numpy(), rtol=1e-12, atol=1e-12)


def test_special_cases():
    rng = np.random.default_rng(4)
    d, inter, r, s = 8, 16, 2, 1.3
    w = _weights(rng, d, inter, r)
    x = rng.normal(0, 1, (7, d))
    # lora_up = 0 on every projection: the base MLP
    w0 = dict(w, b_gate=np.zeros_like(w["b_gate"]), b_up=np.zeros_like(w["b_up"]),
              b_down=np.zeros_like(w["b_down"]))
    base = {k: w[k] for k in ("w_gate", "w_up", "w_down")}
    np.testing.assert_allclose(M.mlp_forward(x, w0, s)["y"], M.mlp_forward(x, base, s)["y"], rtol=0, atol=0)
    # zero gate weights and adapters: silu(0) = 0, so the output is exactly 0
    wz = dict(base, w_gate=np.zeros_like(base["w_gate"]))
    assert np.all(M.mlp_forward(x, wz, s)["y"] == 0.0)
    # one hidden unit, no adapters: y = w_down[:, 0] * silu(x.w_gate) * (x.w_up), written out
    w1 = {"w_gate": rng.normal(0, 1, (1, d)), "w_up": rng.normal(0, 1, (1, d)), "w_down": rng.normal(0, 1, (d, 1))}
    g = x @ w1["w_gate"][0]
    u = x @ w1["w_up"][0]
    want = (g / (1 + np.exp(-g)) * u)[:, None] * w1["w_down"][:, 0][None, :]
    np.testing.assert_allclose(M.mlp_forward(x, w1, s)["y"], want, rtol=1e-12, atol=1e-14)
    # rows are independent: a subset of tokens gives the same rows
    full = M.mlp_forward(x, w, s)["y"]
    np.testing.assert_allclose(M.mlp_forward(x[2:5], w, s)["y"], full[2:5], rtol=0, atol=0)


def test_backward_matches_torch_autograd():
    rng = np.random.default_rng(5)
    d, inter, r, s = 10, 14, 3, 0.9
    w = _weights(rng, d, inter, r)
    x = rng.normal(0, 1, (6, d))
    dy = rng.normal(0, 1, (6, d))
    got = M.mlp_backward(x, w, s, dy)
    xt, t, y = _torch_mlp(x, w, s)
    y.backward(torch.tensor(dy, dtype=torch.float64))
    np.testing.assert_allclose(got["dx"], xt.grad.numpy(), rtol=1e-11, atol=1e-11)
    for name in M.MLP_PROJ:
        np.testing.assert_allclose(got["dA_" + name], t["a_" + name].grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(got["dB_" + name], t["b_" + name].grad.numpy(), rtol=1e-11, atol=1e-11)


def test_backward_directional_finite_differences():
    rng = np.random.default_rng(6)
    d, inter, r, s = 6, 9, 2, 1.1
    w = _weights(rng, d, inter, r)
    x = rng.normal(0, 1, (4, d))
    dy = rng.normal(0, 1, (4, d))
    got = M.mlp_backward(x, w, s, dy)
    h = 1e-6

    def loss(xv, wv):
        return float(np.sum(M.mlp_forward(xv, wv, s)["y"] * dy))

    v = rng.normal(0, 1, x.shape)
    fd = (loss(x + h * v, w) - loss(x - h * v, w)) / (2 * h)
    assert fd == pytest.approx(float(np.sum(got["dx"] * v)), rel=1e-6, abs=1e-8)
    for key in ("a_gate", "b_gate", "a_up", "b_up", "a_down", "b_down"):
        v = rng.normal(0, 1, w[key].shape)
        wp = dict(w, **{key: w[key] + h * v})
        wm = dict(w, **{key: w[key] - h * v})
        fd = (loss(x, wp) - loss(x, wm)) / (2 * h)
        grad = got["d" + key[0].upper() + key[1:]]
        assert fd == pytest.approx(float(np.sum(grad * v)), rel=1e-6, abs=1e-8), key


def test_backward_without_lora_gives_only_dx():
    rng = np.random.default_rng(7)
    w = _weights(rng, 6, 8, 2, lora=False)
    x = rng.normal(0, 1, (3, 6))
    dy = rng.normal(0, 1, (3, 6))
    got = M.mlp_backward(x, w, 0.0, dy)
    assert set(got) == {"dx"}
    xt, _, y = _torch_mlp(x, w, 0.0, lora=False)
    y.backward(torch.tensor(dy, dtype=torch.float64))
    np.testing.assert_allclose(got["dx"], xt.grad.numpy(), rtol=1e-11, atol=1e-11)
