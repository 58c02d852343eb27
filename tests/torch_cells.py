"""The diagonal cells expressed through torch's own GRU / LSTM cells (fp64).

A diagonal cell is D independent scalar cells, one per channel.  A scalar
channel of the diagonal GRU (gates z, r, c; h' = (1-z) h + z c) is exactly
``torch.nn.GRUCell(3, 1)`` with

* input x = (p_z, p_r, p_c), all biases 0,
* weight_ih rows (r | z | n) = (0,1,0 | -1,0,0 | 0,0,1),
* weight_hh = (a_r, -a_z, a_c),

because torch keeps h with weight z_t and mixes in n with (1 - z_t); negating
the z pre-activation turns torch's z_t into our (1 - z).  torch's candidate
n = tanh(W_in x + r * (W_hn h)) is our c = tanh(p_c + a_c r h).

A scalar channel of the diagonal LSTM (gates i, f, o, c; forget bias +1;
state (c, h)) is ``torch.nn.LSTMCell(4, 1)`` with x = (p_i, p_f, p_o, p_c),
weight_ih rows (i | f | g | o) selecting (p_i | p_f | p_c | p_o),
weight_hh = (a_i, a_f, a_c, a_o), bias_ih = (0, 1, 0, 0), bias_hh = 0.

These are independent of the oracle's C code and serve as library pins.
"""
import torch

GRU, LSTM, LINEAR = 1, 2, 0


def gru_cell(a):
    cell = torch.nn.GRUCell(3, 1, bias=True).double()
    with torch.no_grad():
        cell.weight_ih.copy_(torch.tensor([[0.0, 1.0, 0.0], [-1.0, 0.0, 0.0], [0.0, 0.0, 1.0]],
                                          dtype=torch.float64))
        cell.weight_hh.copy_(torch.tensor([[a[1]], [-a[0]], [a[2]]], dtype=torch.float64))
        cell.bias_ih.zero_()
        cell.bias_hh.zero_()
    return cell


def lstm_cell(a):
    cell = torch.nn.LSTMCell(4, 1, bias=True).double()
    with torch.no_grad():
        cell.weight_ih.copy_(torch.tensor([[1.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 0, 1.0], [0, 0, 1.0, 0]],
                                          dtype=torch.float64))
        cell.weight_hh.copy_(torch.tensor([[a[0]], [a[1]], [a[3]], [a[2]]], dtype=torch.float64))
        cell.bias_ih.copy_(torch.tensor([0.0, 1.0, 0.0, 0.0], dtype=torch.float64))
        cell.bias_hh.zero_()
    return cell


def step_fn(cell_id, a):
    """Returns f(s, p) -> s' on fp64 tensors (s: (S,), p: (G,))."""
    if cell_id == GRU:
        m = gru_cell(a)

        def f(s, p):
            return m(p.reshape(1, 3), s.reshape(1, 1)).reshape(1)
        return f
    if cell_id == LSTM:
        m = lstm_cell(a)

        def f(s, p):
            h, c = m(p.reshape(1, 4), (s[1].reshape(1, 1), s[0].reshape(1, 1)))
            return torch.stack([c.reshape(()), h.reshape(())])
        return f

    def f(s, p):
        return p[0] * s + p[1]
    return f


def step_fn_weights(cell_id):
    """f(s, p, a) with the diagonal weights as a differentiable argument."""
    def f(s, p, a):
        if cell_id == GRU:
            w_ih = torch.tensor([[0.0, 1.0, 0.0], [-1.0, 0.0, 0.0], [0.0, 0.0, 1.0]], dtype=torch.float64)
            w_hh = torch.stack([a[1], -a[0], a[2]]).reshape(3, 1)
            z = torch.zeros(3, dtype=torch.float64)
            out = torch._VF.gru_cell(p.reshape(1, 3), s.reshape(1, 1), w_ih, w_hh, z, z)
            return out.reshape(1)
        if cell_id == LSTM:
            w_ih = torch.tensor([[1.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 0, 1.0], [0, 0, 1.0, 0]],
                                dtype=torch.float64)
            w_hh = torch.stack([a[0], a[1], a[3], a[2]]).reshape(4, 1)
            b_ih = torch.tensor([0.0, 1.0, 0.0, 0.0], dtype=torch.float64)
            b_hh = torch.zeros(4, dtype=torch.float64)
            h, c = torch._VF.lstm_cell(p.reshape(1, 4), (s[1].reshape(1, 1), s[0].reshape(1, 1)),
                                       w_ih, w_hh, b_ih, b_hh)
            return torch.stack([c.reshape(()), h.reshape(())])
        return p[0] * s + p[1]
    return f


def unroll_channel(cell_id, p, a, h0):
    """Sequential unroll of one channel: p (T,G), h0 (S,) -> (T,S), fp64."""
    f = step_fn(cell_id, a)
    s = torch.as_tensor(h0, dtype=torch.float64)
    out = []
    with torch.no_grad():
        for t in range(p.shape[0]):
            s = f(s, torch.as_tensor(p[t], dtype=torch.float64))
            out.append(s.clone())
    return torch.stack(out).numpy()
