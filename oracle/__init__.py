"""CPU oracle for the BitLinear hot path.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import anything under oracle/.  The product
package never imports it, and it imports nothing from the product package.
"""
