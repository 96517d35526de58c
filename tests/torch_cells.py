"""Library stand-ins used to pin the CPU oracle: the diagonal GRU / LSTM cells
expressed as ``torch.nn.GRU`` / ``torch.nn.LSTM`` modules in float64.

The diagonal GRU  z = s(u_z + a_z h), r = s(u_r + a_r h),
c = tanh(u_c + a_c r h), h' = (1 - z) h + z c  is torch's GRU with identity
input projections (gate blocks r, z, n), no biases, diagonal hidden weights,
and torch's update gate equal to 1 - z, i.e. its z-block negated:
torch computes h' = (1 - z_t) n + z_t h with z_t = s(-u_z - a_z h) = 1 - z.
The diagonal LSTM (gate order i, f, o, g) is torch's LSTM (gate blocks
i, f, g, o) with identity input projections and diagonal hidden weights.
Nothing here evaluates a cell by hand: torch's own kernels do the arithmetic.
"""
import torch

f64 = torch.float64


def _eye_block(D, G, src):
    """[D, G*D] selector that picks input block ``src``."""
    W = torch.zeros(D, G * D, dtype=f64)
    W[:, src * D:(src + 1) * D] = torch.eye(D, dtype=f64)
    return W


def gru_module(a):
    a = torch.as_tensor(a, dtype=f64)
    D = a.shape[1]
    m = torch.nn.GRU(3 * D, D, bias=False, batch_first=True, dtype=f64)
    with torch.no_grad():
        # torch gate blocks: r, z, n.  Our u blocks: z(0), r(1), c(2).
        m.weight_ih_l0.copy_(torch.cat([_eye_block(D, 3, 1), -_eye_block(D, 3, 0),
                                        _eye_block(D, 3, 2)], 0))
        m.weight_hh_l0.copy_(torch.cat([torch.diag(a[1]), -torch.diag(a[0]),
                                        torch.diag(a[2])], 0))
    return m


def gru_cell_module(a):
    a = torch.as_tensor(a, dtype=f64)
    D = a.shape[1]
    m = torch.nn.GRUCell(3 * D, D, bias=False, dtype=f64)
    g = gru_module(a)
    with torch.no_grad():
        m.weight_ih.copy_(g.weight_ih_l0)
        m.weight_hh.copy_(g.weight_hh_l0)
    return m


def gru_da_from_grad(m, D):
    G = m.weight_hh_l0.grad
    return torch.stack([-torch.diagonal(G[D:2 * D]), torch.diagonal(G[0:D]),
                        torch.diagonal(G[2 * D:3 * D])])


def lstm_module(a):
    a = torch.as_tensor(a, dtype=f64)
    D = a.shape[1]
    m = torch.nn.LSTM(4 * D, D, bias=False, batch_first=True, dtype=f64)
    with torch.no_grad():
        # torch gate blocks: i, f, g, o.  Our u blocks: i(0), f(1), o(2), g(3).
        m.weight_ih_l0.copy_(torch.cat([_eye_block(D, 4, 0), _eye_block(D, 4, 1),
                                        _eye_block(D, 4, 3), _eye_block(D, 4, 2)], 0))
        m.weight_hh_l0.copy_(torch.cat([torch.diag(a[0]), torch.diag(a[1]),
                                        torch.diag(a[3]), torch.diag(a[2])], 0))
    return m


def lstm_cell_module(a):
    a = torch.as_tensor(a, dtype=f64)
    D = a.shape[1]
    m = torch.nn.LSTMCell(4 * D, D, bias=False, dtype=f64)
    g = lstm_module(a)
    with torch.no_grad():
        m.weight_ih.copy_(g.weight_ih_l0)
        m.weight_hh.copy_(g.weight_hh_l0)
    return m


def lstm_da_from_grad(G, D):
    """da [4,D] in our gate order from a [4D, D] weight_hh gradient."""
    return torch.stack([torch.diagonal(G[0:D]), torch.diagonal(G[D:2 * D]),
                        torch.diagonal(G[3 * D:4 * D]), torch.diagonal(G[2 * D:3 * D])])


def gru_run(u, a, h0=None):
    """States h [B,L,D] from torch.nn.GRU."""
    u = torch.as_tensor(u, dtype=f64)
    B, L, G, D = u.shape
    m = gru_module(a)
    hx = None if h0 is None else torch.as_tensor(h0, dtype=f64).reshape(1, B, D)
    with torch.no_grad():
        out, _ = m(u.reshape(B, L, G * D), hx)
    return out


def lstm_run(u, a, c0=None, h0=None):
    """(c, h) [B,L,D] from torch.nn.LSTMCell stepped over L (c is not returned
    per step by nn.LSTM)."""
    u = torch.as_tensor(u, dtype=f64)
    B, L, G, D = u.shape
    m = lstm_cell_module(a)
    h = torch.zeros(B, D, dtype=f64) if h0 is None else torch.as_tensor(h0, dtype=f64)
    c = torch.zeros(B, D, dtype=f64) if c0 is None else torch.as_tensor(c0, dtype=f64)
    cs, hs = [], []
    with torch.no_grad():
        for l in range(L):
            h, c = m(u[:, l].reshape(B, G * D), (h, c))
            cs.append(c)
            hs.append(h)
    return torch.stack(cs, 1), torch.stack(hs, 1)
