"""Derives the cubic used by the softmax's polynomial exp2 (qi21_device.cuh).

Remez exchange for the minimax *relative* error of p(f) ~ 2^f on [-1/2, 1/2]
(degree 3).  Prints the coefficients, their float32 roundings and the maximum
relative error of the rounded polynomial.  Run: python fit_exp2_poly.py
"""
import numpy as np
deg=3
a,b=-0.5,0.5
f=lambda x: np.exp2(x)
# initial reference: Chebyshev extrema
n=deg+2
xs=np.cos(np.pi*np.arange(n)/(n-1))[::-1]*0.5
for it in range(30):
    # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillation)
    A=np.zeros((n,n))
    for i,x in enumerate(xs):
        A[i,:deg+1]=[x**k for k in range(deg+1)]
        A[i,deg+1]=-((-1)**i)*f(x)
    sol=np.linalg.solve(A,f(xs))
    c=sol[:deg+1]; E=sol[deg+1]
    grid=np.linspace(a,b,200001)
    err=(np.polyval(c[::-1],grid)-f(grid))/f(grid)
    # new extrema: pick local extrema of err with alternating signs
    idx=[0]
    for i in range(1,len(grid)-1):
        if (err[i]-err[i-1])*(err[i+1]-err[i])<=0: idx.append(i)
    idx.append(len(grid)-1)
    cand=grid[idx]; ce=err[idx]
    # keep n points with largest |err| alternating
    sel=[]
    for x,e in sorted(zip(cand,ce)):
        if sel and np.sign(e)==np.sign(sel[-1][1]):
            if abs(e)>abs(sel[-1][1]): sel[-1]=(x,e)
        else: sel.append((x,e))
    while len(sel)>n:
        # drop the smaller end
        if abs(sel[0][1])<abs(sel[-1][1]): sel.pop(0)
        else: sel.pop()
    xs=np.array([s[0] for s in sel])
print("coeffs c0..c3:", [float(x) for x in c])
c32=np.array(c,dtype=np.float32)
print("fp32 coeffs:", [float(x) for x in c32], [hex(np.float32(x).view(np.uint32)) for x in c32])
grid=np.linspace(a,b,400001)
err=(np.polyval(c32.astype(np.float64)[::-1],grid)-f(grid))/f(grid)
print("max rel err (exact arithmetic, fp32 coeffs): %.3e = 2^%.2f"%(abs(err).max(), np.log2(abs(err).max())))
