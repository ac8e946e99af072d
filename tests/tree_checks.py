"""Invariants that every outcome of a tree walk satisfies, whatever the
draws: used to check the oracle on random trees and, where the GPU and the
oracle legitimately differ (near-tie decisions), that the GPU's outcome is
still a possible one."""
import numpy as np


def valid_tree_outcome(parent, tokens, V, n, path, out, final_excludes_children=True):
    """parent, tokens: [N] of one sequence; n, path [N], out [N]: its result.

    The path starts at the root and steps from each node to one of its
    children (a node whose parent is the previous path node), committing that
    child's token, which must be a real token; the entries after the path and
    after the drawn token are -1; the drawn token is a real token and, in the
    stochastic rule, none of the final node's valid children's tokens (they
    were all rejected, so they left the draw's support)."""
    parent = np.asarray(parent)
    tokens = np.asarray(tokens)
    N = len(parent)
    if not (0 <= n < N) or path[0] != 0:
        return False
    for i in range(1, n + 1):
        j = int(path[i])
        if not (0 < j < N) or parent[j] != path[i - 1] or not (0 <= tokens[j] < V):
            return False
        if out[i - 1] != tokens[j]:
            return False
    if (np.asarray(path[n + 1:]) != -1).any() or (np.asarray(out[n + 1:]) != -1).any():
        return False
    if not (0 <= out[n] < V):
        return False
    if final_excludes_children:
        u = int(path[n])
        kids = {int(tokens[j]) for j in range(u + 1, N)
                if parent[j] == u and 0 <= tokens[j] < V}
        if int(out[n]) in kids:
            return False
    return True
